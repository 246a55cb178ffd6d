/*
 * csld.h -- C ABI of libcsld.so: the decode hot path of hybrid compressed attention
 * (CSA + HCA) on NVIDIA B200 (sm_100a).
 *
 * The operations follow the pages about DeepSeek-V4:
 *  [HF]  "DeepSeek-V4: a million-token context that agents can actually use" (Korean rendering
 *        of the Hugging Face blog): CSA paragraph and Figure 3 caption (4x softmax-gated pooling
 *        with a learned positional bias; FP4 ReLU-scored multi-head lightning indexer; top-k
 *        compressed blocks per query; sliding-window branch), HCA paragraph and Figure 4 caption
 *        (128x compression, dense attention over the compressed stream, same window branch),
 *        storage paragraph (KV mostly FP8, RoPE dims BF16, indexer FP4).
 *  [VEL] velog.io "DeepSeek V4 paper review": "core technique 1: CSA", "core technique 2: HCA",
 *        and the KV-cache-layout section (compressed caches, a separate sliding-window state,
 *        a separately kept uncompressed tail).
 *
 * Conventions for every call:
 *  - All array pointers are DEVICE pointers owned by the caller; the library allocates nothing.
 *    Scratch ("workspace") is caller-provided; its size comes from the *_workspace_size query.
 *  - bf16 values are passed as their raw 16-bit patterns (uint16_t).
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).  Every
 *    call only enqueues work on `stream` and returns; nothing synchronises the host.
 *  - Arguments are validated on the host before anything is launched; on a bad argument the
 *    call returns a non-zero csld_status, launches nothing and leaves a message in
 *    csld_last_error() (thread-local).  A failed launch returns CSLD_ERR_CUDA.
 *  - Conditions only the device can see (a top-k index that is not a visible entry, a full
 *    compressed cache) are never turned into traps: the kernel skips the offending item and
 *    ORs a flag into the caller's device error word `err` (may be NULL), see CSLD_DEVERR_*.
 *  - Shapes fixed by the format: D = 512 (448 "nope" dims stored E4M3 + 64 RoPE dims stored
 *    bf16, one shared KV head whose 512-d entry is both key and value), 16 query heads per KV
 *    head in the decode kernel, 4 indexer heads x 64 dims.
 */
#ifndef CSLD_H
#define CSLD_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define CSLD_API __attribute__((visibility("default")))
#else
#define CSLD_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define CSLD_ABI_VERSION 1

#define CSLD_DIM 512            /* entry / head dimension */
#define CSLD_DIM_NOPE 448       /* dims 0..447 stored as E4M3 (scale 1, RNE, saturating) */
#define CSLD_DIM_ROPE 64        /* dims 448..511 stored as bf16 */
#define CSLD_ENTRY_BYTES 576    /* 448 E4M3 bytes followed by 64 little-endian bf16 */
#define CSLD_HEADS 16           /* query heads sharing the KV head (decode kernel) */
#define CSLD_IDX_HEADS 4        /* lightning-indexer heads */
#define CSLD_IDX_DIM 64         /* lightning-indexer dims per head (one key shared by the heads) */
#define CSLD_IKEY_BYTES 32      /* 64 E2M1 codes, element 2i in the low nibble of byte i,
                                   stored with halves swapped when bit 2 of the entry index
                                   is set (see "Indexer key storage" below) */
#define CSLD_IKEY_SCALES 2      /* fp32 power-of-two scale per group of 32 codes */
#define CSLD_MAX_RATIO 128      /* tokens per compressed entry: 1..128 (CSA 4, HCA 128) */
#define CSLD_MAX_WINDOW 1024    /* sliding-window length in raw tokens: 0..1024 */
#define CSLD_MAX_TOPK 2048      /* indexer top-k: 1..2048 */

typedef enum csld_status {
    CSLD_OK = 0,
    CSLD_ERR_ARG = 1,          /* null pointer or out-of-range scalar */
    CSLD_ERR_SHAPE = 2,        /* inconsistent sizes */
    CSLD_ERR_ALIGN = 3,        /* a pointer or stride is not 16-byte aligned */
    CSLD_ERR_CAPACITY = 4,     /* a size exceeds a stated maximum or the cache capacity */
    CSLD_ERR_CUDA = 5,         /* a CUDA runtime error (launch failure, no device, ...) */
    CSLD_ERR_UNSUPPORTED = 6,  /* a shape the library does not implement (e.g. heads != 16) */
    CSLD_ERR_WORKSPACE = 7     /* workspace pointer NULL or smaller than required */
} csld_status;

/* Device error word flags (ORed into `err` by kernels). */
#define CSLD_DEVERR_CAPACITY 1u     /* kv_cache_append: entry index >= capacity; token dropped */
#define CSLD_DEVERR_BAD_INDEX 2u    /* hybrid_decode_attention: a top-k index was not visible */
#define CSLD_DEVERR_SEQ_LEN 4u      /* a seq_len < 0; that sequence was treated as empty */
#define CSLD_DEVERR_TIMEOUT 8u      /* a bounded wait for an asynchronous copy gave up */

CSLD_API int csld_abi_version(void);
CSLD_API const char* csld_last_error(void);
CSLD_API const char* csld_status_string(csld_status s);

/* ----------------------------------------------------------------------------------------
 * Indexer key storage.  Entry s of a key array ([..][cap][32] u8) holds the 64 E2M1 codes of
 * its key: logical byte c (elements 2c and 2c+1; bytes 0..15 are group 0, 16..31 group 1)
 * is stored at byte  s*32 + (c XOR 16*((s >> 2) & 1)),  i.e. the two 16-byte halves trade
 * places in entries 4..7 of every 8.  That is the 32-byte-swizzled K-major operand layout of
 * the tensor cores, so a run of entries that starts at a multiple of 8 is copied into shared
 * memory byte for byte and used as an MMA operand as it lands.  csld_compress and
 * kv_cache_append write this layout and indexer_topk reads it; the swap is its own inverse.
 * The scales ([..][cap][2] f32, group 0 then group 1) are not permuted.
 * ---------------------------------------------------------------------------------------- */
/* ----------------------------------------------------------------------------------------
 * Prefill compression ([HF] CSA paragraph, Figure 3; HCA paragraph, Figure 4).
 * For one sequence of T raw tokens, block s = tokens s*m .. s*m+m-1 becomes entry s:
 *   a_j = gate[s*m+j] + pos_bias[j];  w = softmax(a);  c = sum_j w_j * raw[s*m+j]   (fp32)
 *   kv_out[s]  = E4M3(c[0:448]) || bf16(c[448:512])                                 (RNE)
 * and, when w_idx != NULL (CSA layers), the lightning-indexer key
 *   u = c . W_I  (bf16 operands, fp32 accumulation),  ikey_out[s] = E2M1 codes of u / sigma_g
 *   (stored as "Indexer key storage" describes),
 *   iscale_out[s][g] = sigma_g = smallest power of two with max|u in group g| <= 6 sigma_g.
 * The trailing T mod m tokens form no entry.
 *   raw        [T][512] bf16     gate [T] f32     pos_bias [m] f32     w_idx [512][64] f32
 *   kv_out     [T/m][576] u8     ikey_out [T/m][32] u8     iscale_out [T/m][2] f32
 * raw, kv_out, ikey_out must be 16-byte aligned.  1 <= ratio <= 128.
 * csa_compress = csld_compress with ratio 4 and the indexer key; hca_compress = ratio 128
 * without it.
 * -------------------------------------------------------------------------------------- */
CSLD_API csld_status csld_compress(const uint16_t* raw, const float* gate, const float* pos_bias,
                          int ratio, const float* w_idx, int64_t T, uint8_t* kv_out,
                          uint8_t* ikey_out, float* iscale_out, void* stream);
CSLD_API csld_status csa_compress(const uint16_t* raw, const float* gate, const float* pos_bias,
                         const float* w_idx, int64_t T, uint8_t* kv_out, uint8_t* ikey_out,
                         float* iscale_out, void* stream);
CSLD_API csld_status hca_compress(const uint16_t* raw, const float* gate, const float* pos_bias,
                         int64_t T, uint8_t* kv_out, void* stream);

/* ----------------------------------------------------------------------------------------
 * Per-channel gated compression -- the other plain reading of "softmax-gated pooling with a
 * learned positional bias" ([HF] CSA paragraph; Figure 3 caption; HCA paragraph): a gate
 * logit for every token AND dimension and a bias for every block slot and dimension.  Each
 * dimension d of entry s pools its own softmax:
 *   a_j = gate[s*m+j][d] + pos_bias[j][d],  w = softmax_j(a),  c_d = sum_j w_j raw[s*m+j][d],
 * then the entry and (w_idx != NULL) the FP4 indexer key exactly as csld_compress writes them
 * (the key projected from bf16 operands with fp32 accumulation).  With gate and bias equal
 * across dimensions this is csld_compress.
 *   gate [T][512] f32, pos_bias [ratio][512] f32; others as for csld_compress; raw, gate,
 *   pos_bias, kv_out, ikey_out 16-byte aligned.
 * -------------------------------------------------------------------------------------- */
CSLD_API csld_status csld_compress_channel(const uint16_t* raw, const float* gate, const float* pos_bias,
                                           int ratio, const float* w_idx, int64_t T, uint8_t* kv_out,
                                           uint8_t* ikey_out, float* iscale_out, void* stream);

/* ----------------------------------------------------------------------------------------
 * RoPE at compressed positions -- a layout variant of the storage paragraph ([HF]: each
 * entry keeps its RoPE dims in bf16), where the library applies the rotary position encoding
 * itself instead of storing the RoPE dims as given.  raw's dims 448..511 are taken BEFORE
 * rotary encoding.  Entry s (tokens s*m .. s*m+m-1 of raw) is pooled exactly as by
 * csld_compress; then its dims 448..511 are rotated at the position of its block's last token,
 *   p_s = pos0 + (s+1)*ratio - 1,
 * pair i = dims (448 + 2i, 449 + 2i), i = 0..31, turned by the angle p_s * rope_base^(-i/32)
 * (RoFormer), before the bf16 rounding of the entry and before the indexer key is projected
 * (the key is the FP4 code of the rotated vector times W_I).  pos0 = position of raw[0],
 * 0 <= pos0 <= 2^40; rope_base finite and > 1 (10000 in the usual setting).  The query's RoPE
 * dims are the caller's to rotate, at the query's own position.  Arguments, layouts, alignment
 * and errors otherwise as csld_compress; rotations are computed in double and rounded to fp32,
 * so the stored bf16 values agree with an exact rotation to within one bf16 step.
 * -------------------------------------------------------------------------------------- */
CSLD_API csld_status csld_compress_rope(const uint16_t* raw, const float* gate, const float* pos_bias,
                                        int ratio, const float* w_idx, int64_t T, int64_t pos0,
                                        double rope_base, uint8_t* kv_out, uint8_t* ikey_out,
                                        float* iscale_out, void* stream);

/* ----------------------------------------------------------------------------------------
 * One layer's KV-cache state for B sequences ([VEL] KV-cache-layout section: compressed
 * cache, separate sliding-window state, separately kept uncompressed tail).  A host struct of
 * device pointers; the caller owns all of it.
 *   comp_kv   [B][capacity][576]  compressed entries (entry s = tokens s*m .. s*m+m-1)
 *   ikeys     [B][capacity][32]   indexer key codes     (has_indexer != 0; else NULL)
 *   iscales   [B][capacity][2]    indexer key scales    (has_indexer != 0; else NULL)
 *   win_kv    [B][window][576]    ring of the last `window` raw tokens, token t at slot t mod W
 *   tail_kv   [B][ratio][512]     bf16 raw tokens of the block being filled, token t at t mod m
 *   tail_gate [B][ratio]          their gate logits
 *   seq_len   [B]                 raw tokens so far (int32, device)
 *   pos_bias  [ratio]             positional bias of the pooling
 *   w_idx     [512][64]           indexer projection (has_indexer != 0)
 * capacity must be even (16-byte alignment of the per-sequence scale arrays).
 * -------------------------------------------------------------------------------------- */
typedef struct csld_layer_cache {
    int32_t ratio;
    int32_t window;
    int32_t batch;
    int32_t has_indexer;
    int64_t capacity;
    uint8_t* comp_kv;
    uint8_t* ikeys;
    float* iscales;
    uint8_t* win_kv;
    uint16_t* tail_kv;
    float* tail_gate;
    int32_t* seq_len;
    const float* pos_bias;
    const float* w_idx;
} csld_layer_cache;

/* Decode-time append of ONE raw token per sequence ([VEL] KV-cache layout; [HF] Figures 3-4).
 * For sequence b with t = seq_len[b]:  window slot t mod W <- entry(kv_new[b]);
 * tail slot t mod m <- (kv_new[b], gate_new[b]);  when (t+1) mod m == 0 the m tail tokens are
 * pooled (same arithmetic as csld_compress) into entry t/m (+ indexer key);  seq_len[b] = t+1.
 * If entry t/m would not fit in capacity, nothing of sequence b changes and
 * CSLD_DEVERR_CAPACITY is ORed into *err.
 *   kv_new [B][512] bf16, gate_new [B] f32, err: device int32 or NULL. */
CSLD_API csld_status kv_cache_append(const csld_layer_cache* cache, const uint16_t* kv_new,
                            const float* gate_new, int32_t* err, void* stream);

/* Prefill of all B sequences with T raw tokens each (raw [B][T][512], gate [B][T]): writes
 * entries 0..T/m-1 (+ keys), the window ring with the last min(W, T) tokens, the tail with the
 * last T mod m tokens, and sets seq_len[b] = T.  Equivalent to T calls of kv_cache_append on
 * an empty cache.  Requires T/m <= capacity. */
CSLD_API csld_status kv_cache_prefill(const csld_layer_cache* cache, const uint16_t* raw,
                             const float* gate, int64_t T, void* stream);

/* kv_cache_append / kv_cache_prefill with RoPE at compressed positions (see csld_compress_rope):
 * the tokens' dims 448..511 arrive before rotary encoding; token t's window entry holds them
 * rotated at position t, and a completed entry s is rotated at position (s+1)*ratio - 1, the
 * token that completes it (the tail keeps the tokens as given).  Positions count from 0 at the
 * first token of each sequence.  rope_base finite and > 1; a cache must be filled by one kind
 * of call throughout.  Otherwise as kv_cache_append / kv_cache_prefill. */
CSLD_API csld_status kv_cache_append_rope(const csld_layer_cache* cache, const uint16_t* kv_new,
                                          const float* gate_new, double rope_base, int32_t* err,
                                          void* stream);
CSLD_API csld_status kv_cache_prefill_rope(const csld_layer_cache* cache, const uint16_t* raw,
                                           const float* gate, int64_t T, double rope_base, void* stream);

/* ----------------------------------------------------------------------------------------
 * Per-head indexer keys -- a layout variant of the lightning indexer ([HF] CSA paragraph:
 * "FP4, ReLU-scored multi-head dot product"), where every one of the 4 indexer heads has its own
 * projection and its own key per entry, instead of one key shared by the heads:
 *   u_h = c . W_h (bf16 operands, fp32 accumulation),  w_idx [512][4][64] f32 (W_h[d][j] at
 *   d*256 + h*64 + j);  key h = FP4 of u_h exactly as the shared key is quantised.
 * Stored layout: ikey_out / ikeys [entries][128] u8 -- the four heads' 32 code bytes in head
 * order, and within each 8-entry block the 16-byte chunk c (c = 2*head + group) of entry s
 * stored at chunk c ^ (s mod 8) (the tensor cores' 128-byte swizzle); iscale_out / iscales
 * [entries][4][2] f32.  T/ratio entries; 16-byte alignment as for csld_compress.
 *   csld_compress_perhead, kv_cache_prefill_perhead, kv_cache_append_perhead: as csld_compress,
 *     kv_cache_prefill, kv_cache_append with such keys (the cache's ikeys [B][capacity][128],
 *     iscales [B][capacity][4][2], w_idx [512][4][64]);
 *   indexer_topk_perhead: as indexer_topk_multi (Q query tokens per sequence, 1 <= Q <=
 *     CSLD_MULTI_MAX_Q; Q = 1 is the decode step), head h's dot taken against key h, with the
 *     same fp32 operation order; workspace csld_indexer_multi_workspace_size(B, Q, cap).
 * -------------------------------------------------------------------------------------- */
CSLD_API csld_status csld_compress_perhead(const uint16_t* raw, const float* gate, const float* pos_bias,
                                           int ratio, const float* w_idx, int64_t T, uint8_t* kv_out,
                                           uint8_t* ikey_out, float* iscale_out, void* stream);
CSLD_API csld_status kv_cache_prefill_perhead(const csld_layer_cache* cache, const uint16_t* raw,
                                              const float* gate, int64_t T, void* stream);
CSLD_API csld_status kv_cache_append_perhead(const csld_layer_cache* cache, const uint16_t* kv_new,
                                             const float* gate_new, int32_t* err, void* stream);
CSLD_API csld_status indexer_topk_perhead(const uint8_t* ikeys, const float* iscales, int64_t cap,
                                          const int32_t* seq_len, int ratio, const float* q_idx,
                                          const float* head_w, int B, int Q, int k, int32_t* topk_out,
                                          void* ws, size_t ws_bytes, int32_t* err, void* stream);

/* ----------------------------------------------------------------------------------------
 * Scaled FP8 entries -- a layout variant of the storage paragraph ([HF]: entries FP8 except the
 * RoPE dims in bf16), with one positive scale kv_scale (sigma) per layer cache: an entry's (and
 * a window entry's) 448 FP8 dims hold E4M3(x / sigma), RNE, saturating at +-448, and stand for
 * sigma times their code value; the 64 bf16 RoPE dims are not scaled; the indexer key is
 * projected from the unscaled pooled vector.  A small sigma keeps values below E4M3's
 * subnormals, a large one values above 448.  2^-60 <= kv_scale <= 2^60.
 *   csld_compress_scaled, kv_cache_prefill_scaled, kv_cache_append_scaled: as csld_compress,
 *     kv_cache_prefill, kv_cache_append, writing scaled entries (a cache must be filled with
 *     one sigma throughout);
 *   hybrid_decode_attention_scaled: as hybrid_decode_attention over such entries -- the keys
 *     and values are the decoded entries with their FP8 dims times kv_scale.
 * The device multiplies by 1 / sigma in fp32 before rounding, so an E4M3 code may differ by one
 * step from the exact quotient's where that lands near a rounding midpoint.
 * -------------------------------------------------------------------------------------- */
CSLD_API csld_status csld_compress_scaled(const uint16_t* raw, const float* gate, const float* pos_bias,
                                          int ratio, const float* w_idx, int64_t T, float kv_scale,
                                          uint8_t* kv_out, uint8_t* ikey_out, float* iscale_out,
                                          void* stream);
CSLD_API csld_status kv_cache_prefill_scaled(const csld_layer_cache* cache, const uint16_t* raw,
                                             const float* gate, int64_t T, float kv_scale, void* stream);
CSLD_API csld_status kv_cache_append_scaled(const csld_layer_cache* cache, const uint16_t* kv_new,
                                            const float* gate_new, float kv_scale, int32_t* err,
                                            void* stream);

/* ----------------------------------------------------------------------------------------
 * Lightning indexer + top-k ([HF] CSA paragraph: "FP4, ReLU-scored multi-head dot product"
 * picks the top-k compressed blocks per query; [VEL] core technique 1).
 * For sequence b, the visible entries are s < n_b = min(seq_len[b] / ratio, cap).  The query
 * q_idx[b][h] (fp32) is quantised to FP4 exactly like the keys (E2M1, power-of-two scale per
 * 32); per entry and head the two FP4 vectors give an exact dot d; the score is
 *   e_s = sum_h head_w[b][h] * max(d_h, 0)
 * formed in fp32 in the fixed order  e = w0*r0; e = fma(w1,r1,e); e = fma(w2,r2,e);
 * e = fma(w3,r3,e)  with  d_h = fma(I1, s1, I0*s0),  I_g the integer group dots (x4) and
 * s_g = (qscale_g * kscale_g) * 0.25.  The min(k, n_b) entries with the largest (score,
 * -index) are written to topk_out[b] in ascending index order, followed by -1 padding.
 *   ikeys [B][cap][32] u8, iscales [B][cap][2] f32, seq_len [B] i32, q_idx [B][4][64] f32,
 *   head_w [B][4] f32, topk_out [B][k] i32.  ikeys in the stored layout of "Indexer key
 *   storage".  cap even, 2 <= cap <= 2^30; ikeys and iscales 16-byte aligned; 1 <= k <= 2048.
 * Workspace: csld_indexer_workspace_size(B, cap, k) bytes, 256-byte aligned, zero-filled once
 * before its first use (it holds per-sequence selection state, in two sets that alternate
 * between calls: each call clears the set the next call will use); calls that share one
 * workspace must not overlap on the GPU.  After a call that reported CSLD_DEVERR_TIMEOUT,
 * zero it again.  err: device error word or NULL. */
CSLD_API size_t csld_indexer_workspace_size(int B, int64_t cap, int k);
CSLD_API csld_status indexer_topk(const uint8_t* ikeys, const float* iscales, int64_t cap,
                         const int32_t* seq_len, int ratio, const float* q_idx,
                         const float* head_w, int B, int k, int32_t* topk_out, void* ws,
                         size_t ws_bytes, int32_t* err, void* stream);

/* ----------------------------------------------------------------------------------------
 * Multi-query lightning indexer ([HF] CSA paragraph; layer-pattern paragraph: the
 * multi-token-prediction block runs several query tokens per step).  Q query tokens per
 * sequence -- the Q newest tokens: query j of sequence b stands at raw position
 * p = seq_len[b] - Q + j and sees the entries s < min((p + 1) / ratio, cap) -- are scored in
 * one pass over the key cache (the tensor cores take all Q queries as one operand), and each
 * gets its own exact top-k.  Scores, ties and output order are those of indexer_topk for that
 * query alone, so topk_out[b][j] equals indexer_topk with seq_len = p + 1 and query j.
 *   ikeys / iscales as for indexer_topk, q_idx [B][Q][4][64] f32, head_w [B][Q][4] f32,
 *   topk_out [B][Q][k] i32 (ascending, -1 padded).  1 <= Q <= CSLD_MULTI_MAX_Q, 1 <= k <= 2048.
 * Workspace: csld_indexer_multi_workspace_size(B, Q, cap) bytes (the Q score arrays and their
 * histograms), 256-byte aligned, zero-filled once before its first use; each call leaves it
 * ready for the next.  Calls that share one workspace must not overlap on the GPU; after a call
 * that reported CSLD_DEVERR_TIMEOUT, zero it again.
 * ---------------------------------------------------------------------------------------- */
#define CSLD_MULTI_MAX_Q 8
CSLD_API size_t csld_indexer_multi_workspace_size(int B, int Q, int64_t cap);
CSLD_API csld_status indexer_topk_multi(const uint8_t* ikeys, const float* iscales, int64_t cap,
                                        const int32_t* seq_len, int ratio, const float* q_idx,
                                        const float* head_w, int B, int Q, int k, int32_t* topk_out,
                                        void* ws, size_t ws_bytes, int32_t* err, void* stream);

/* ----------------------------------------------------------------------------------------
 * Hybrid decode attention ([HF] CSA paragraph + Figure 3: attention over the selected entries
 * plus a sliding-window branch; HCA paragraph + Figure 4: dense attention over every
 * compressed entry plus the same window branch).
 * For sequence b (n = seq_len[b], n_vis = min(n / ratio, cap)) the key set is
 *   { comp_kv[b][s] : s in topk[b], s >= 0 }   (sparse mode, topk != NULL), or
 *   { comp_kv[b][s] : s < n_vis }                (dense mode, topk == NULL),
 * together with { win_kv[b][t mod W] : max(0, n-W) <= t < n }.  Keys = values = the decoded
 * 512-vectors; for each head h: out[b][h] = softmax(scale * q[b][h] . K^T) V, one joint
 * softmax over the union; lse_out[b][h] = natural log of the softmax denominator in logit
 * units.  An empty key set gives out = 0 and lse = -inf.
 *   q [B][heads][512] bf16 (heads == 16), comp_kv [B][cap][576], topk [B][k] i32 or NULL,
 *   win_kv [B][W][576], seq_len [B] i32, out [B][heads][512] f32, lse_out [B][heads] f32 or NULL.
 * out and lse_out are written with plain stores, so they may also be pinned host memory mapped
 * into the device's address space (the result then lands on the host without a separate copy).
 * comp_kv, win_kv must be 16-byte aligned.  Workspace: csld_attention_workspace_size(...).
 * -------------------------------------------------------------------------------------- */
CSLD_API size_t csld_attention_workspace_size(int B, int heads, int64_t cap, int k, int W);
CSLD_API csld_status hybrid_decode_attention(const uint16_t* q, int heads, const uint8_t* comp_kv,
                                    int64_t cap, int ratio, const int32_t* topk, int k,
                                    const uint8_t* win_kv, int W, const int32_t* seq_len, int B,
                                    float scale, float* out, float* lse_out, void* ws,
                                    size_t ws_bytes, int32_t* err, void* stream);
/* hybrid_decode_attention over scaled FP8 entries (see csld_compress_scaled): the query's FP8
 * part is multiplied by kv_scale before it meets the codes, and the output's FP8 dims by
 * kv_scale at the end.  2^-60 <= kv_scale <= 2^60; otherwise as hybrid_decode_attention. */
CSLD_API csld_status hybrid_decode_attention_scaled(const uint16_t* q, int heads, const uint8_t* comp_kv,
                                                    int64_t cap, int ratio, const int32_t* topk, int k,
                                                    const uint8_t* win_kv, int W, const int32_t* seq_len,
                                                    int B, float scale, float kv_scale, float* out,
                                                    float* lse_out, void* ws, size_t ws_bytes, int32_t* err,
                                                    void* stream);

/* ----------------------------------------------------------------------------------------
 * Multi-query decode attention ([HF] layer-pattern paragraph: the multi-token-prediction block
 * runs several query tokens per step; CSA / HCA paragraphs as above).  Q query tokens per
 * sequence -- the Q newest: query j of sequence b stands at raw position seq_len[b] - Q + j --
 * share one launch over the cache; query j sees the first seq_len[b] - Q + 1 + j tokens: the
 * compressed entries they complete (dense mode) or its own top-k row (sparse mode), and the W
 * newest of them through the window ring.  Each (b, j) gets exactly what hybrid_decode_attention
 * gives that query alone.
 *   q [B][Q][heads][512] bf16, topk [B][Q][k] i32 or NULL, out [B][Q][heads][512] f32,
 *   lse_out [B][Q][heads] f32 or NULL; the window ring win_kv [B][W_ring][576] holds token t at
 *   slot t mod W_ring, W_ring >= W + Q - 1 (so the oldest query's window is still in it: a
 *   layer cache whose window is W_ring, fed by kv_cache_append, keeps it that way).
 *   1 <= Q <= CSLD_MULTI_MAX_Q, B * Q <= 65535.
 * Workspace: csld_attention_workspace_size(B * Q, heads, cap, k, W).  Other rules as for
 * hybrid_decode_attention.
 * -------------------------------------------------------------------------------------- */
CSLD_API csld_status hybrid_decode_attention_multi(const uint16_t* q, int heads, const uint8_t* comp_kv,
                                                   int64_t cap, int ratio, const int32_t* topk, int k,
                                                   const uint8_t* win_kv, int W_ring, int W,
                                                   const int32_t* seq_len, int B, int Q, float scale,
                                                   float* out, float* lse_out, void* ws,
                                                   size_t ws_bytes, int32_t* err, void* stream);

/* ----------------------------------------------------------------------------------------
 * hybrid_decode_attention_static -- the same computation as hybrid_decode_attention, for
 * callers that cannot allocate device memory on their call path.  The pages have no
 * counterpart to this entry point: it exists for integration only.  Examples are a plug-in
 * whose host framework owns every device allocation and hands it only inputs and outputs,
 * and a decode loop that must not call the CUDA allocator between steps (an allocation can
 * synchronise the device or fail under memory pressure).
 *
 * Instead of a caller workspace it uses one fixed scratch array of CSLD_STATIC_SCRATCH_BYTES
 * inside the library.  Every GPU that loads libcsld.so keeps that array until the process
 * exits.  It allocates nothing:
 *  - The first call on a device (with that device current) looks up the array's device
 *    address once and keeps it for the life of the process. Make that first call before any
 *    stream capture.  A cudaDeviceReset on that device invalidates the kept address: do not
 *    call this entry point on a device after resetting it.
 *  - A call that would need more scratch than the array holds returns CSLD_ERR_CAPACITY and
 *    launches nothing (the need is about B * min(#SMs/B, tiles) * 16 * 2056 bytes; batches up
 *    to ~250 sequences fit).
 *  - All calls share the array, and it keeps the last call's contents. Nothing in it needs to
 *    start at zero, but two calls that overlap on the GPU (different streams without ordering,
 *    or different host threads) race on it and corrupt each other's results.
 * Arguments, layouts, results and error handling are those of hybrid_decode_attention.
 * -------------------------------------------------------------------------------------- */
#define CSLD_STATIC_SCRATCH_BYTES (8u * 1024u * 1024u)
CSLD_API csld_status hybrid_decode_attention_static(const uint16_t* q, int heads,
                                                    const uint8_t* comp_kv, int64_t cap, int ratio,
                                                    const int32_t* topk, int k,
                                                    const uint8_t* win_kv, int W,
                                                    const int32_t* seq_len, int B, float scale,
                                                    float* out, float* lse_out, int32_t* err,
                                                    void* stream);

/* ----------------------------------------------------------------------------------------
 * Context-parallel decode: one sequence's compressed cache split over R GPUs, rank r holding
 * the contiguous entries [lo_r, lo_r + n_r) of every sequence (the window ring and the tail on
 * one rank).  ([HF] CSA paragraph: the indexer picks the top-k compressed blocks per query; HCA
 * paragraph: dense attention over the compressed stream.  The split is this library's; the
 * pages run everything on one device.)  A decode step on rank r:
 *   1. indexer_topk on the local keys -> local selection;  indexer_rescore -> their scores;
 *      the caller all-gathers (score, local index) over the ranks into [R][B][k];
 *   2. csld_topk_merge -> the global top-k, written as this rank's local indices;
 *   3. hybrid_decode_attention on the local cache with that selection (sparse mode; dense mode
 *      for HCA layers) -> (out_r, lse_r); the caller all-gathers them into [R][B][16][512] and
 *      [R][B][16];
 *   4. csld_lse_merge -> the step's output.
 * Because the top-k of a union is the top-k of the union of the parts' top-k, and a softmax over
 * a union of key sets is the log-sum-exp combination of the parts, the result is the single-GPU
 * one: the same selection, and the same output up to fp32 rounding.
 *
 * indexer_rescore: scores_out[b][j] = the fp32 score (same quantisation and operation order as
 * indexer_topk) of entry sel[b][j] of sequence b, or -inf where sel[b][j] < 0 or >= cap.
 *   ikeys / iscales as for indexer_topk (stored layout, cap even, iscales 16-byte aligned),
 *   q_idx [B][4][64] f32, head_w [B][4] f32, sel [B][k] i32, scores_out [B][k] f32.
 * csld_topk_merge: cand_scores [R][B][k] f32 and cand_idx [R][B][k] i32 (indices local to rank
 *   r's range, -1 = none), rank_lo [R] i64 (device: where rank r's range starts) -> topk_out[b] =
 *   the min(k, #candidates) best candidates of sequence b by (score desc, global index asc), in
 *   ascending index order, each written as global - lo when lo <= global < lo + n_local and as
 *   -1 otherwise; -1 padded.  R * k <= 16384; global indices below 2^31 - 1.
 * csld_lse_merge: outs [R][B][heads][512] f32, lses [R][B][heads] f32 (natural log; -inf =
 *   empty part) -> out [B][heads][512] = sum_r exp(lses_r - L) outs_r, lse_out [B][heads] = L
 *   = log sum_r exp(lses_r) (may be NULL).  heads == 16; outs and out 16-byte aligned.
 * All three only enqueue kernels on `stream`; the all-gathers between them are the caller's
 * (NCCL over NVLink in the Python binding).
 * ---------------------------------------------------------------------------------------- */
CSLD_API csld_status indexer_rescore(const uint8_t* ikeys, const float* iscales, int64_t cap,
                                     const float* q_idx, const float* head_w, const int32_t* sel, int B,
                                     int k, float* scores_out, void* stream);
CSLD_API csld_status csld_topk_merge(const float* cand_scores, const int32_t* cand_idx,
                                     const int64_t* rank_lo, int R, int B, int k, int64_t lo,
                                     int64_t n_local, int32_t* topk_out, void* stream);
CSLD_API csld_status csld_lse_merge(const float* outs, const float* lses, int R, int B, int heads,
                                    float* out, float* lse_out, void* stream);

/* ----------------------------------------------------------------------------------------
 * csld_stage -- copies `bytes` from src to dst with a kernel on `stream`.  The pages have no
 * counterpart to this entry point: it serves callers that bring a decode step's inputs from
 * the host.  dst and src may each be device memory or pinned host memory mapped into the
 * device's address space (with unified addressing, any cudaHostAlloc / cudaMallocHost
 * allocation).  As a kernel it chains directly to the decode kernel after it and may start
 * while the kernel before it finishes (dst is written only after that kernel has completed),
 * where a copy-engine transfer between two kernels costs a round trip through the copy engine.
 * dst and src 16-byte aligned, bytes a multiple of 16; the two ranges must not overlap.
 * ---------------------------------------------------------------------------------------- */
CSLD_API csld_status csld_stage(void* dst, const void* src, size_t bytes, void* stream);

/* ----------------------------------------------------------------------------------------
 * Test hook (no counterpart on the pages): the indexer's cooperative kernel waits, with a bound
 * of about half a second each, for the CTAs of a sequence: until their level-1 histogram holds
 * every key, and at up to three cross-CTA barriers.  This call adds `extra` to that key total and
 * to every barrier target of the calls that follow (0 restores normal use), so that a test can
 * make those waits run out and check the recovery: the kernel returns,
 * CSLD_DEVERR_TIMEOUT is set in the error word, and the workspace must be zero-filled again
 * before the next call.  Process-wide; not for production use.
 * ---------------------------------------------------------------------------------------- */
CSLD_API void csld_test_set_barrier_extra(int extra);

#ifdef __cplusplus
}
#endif
#endif /* CSLD_H */
