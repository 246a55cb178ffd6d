// Hybrid decode attention on the 5th-generation tensor cores (tcgen05).
//
// Source: "DeepSeek-V4: a million-token context that agents can actually use" -- CSA paragraph
// and Figure 3 caption (each query attends to its top-k compressed blocks; a sliding-window
// branch covers the most recent uncompressed tokens), HCA paragraph and Figure 4 caption
// (every query attends densely to all compressed blocks; the same window branch), storage
// paragraph (entries FP8 except the RoPE dims in bf16); velog.io paper review, core
// techniques 1-2.  Keys and values are the same 576-byte entry (448 E4M3 dims + 64 bf16 RoPE
// dims); 16 query heads share it; one softmax runs over {selected or all visible entries} +
// {window tokens}.
//
// One CTA = one split of one sequence's key list, walked in tiles of 96 entries; 16 warps.
//  - Warps 0-3 bring a tile in: five 128-byte column blocks of every entry (bytes 0, 128, 256,
//    384 and 448 -- the last one is the RoPE part), each block [96 entries][128 B] with the
//    128-byte swizzle, into one of three tile buffers, so copies run up to two tiles ahead of
//    the PV that frees a buffer.  (The QK MMA has 128 rows: it also reads the 32 rows after a
//    block, whose scores are never used.)  Contiguous tiles take one TMA box copy per block;
//    other tiles are gathered entry by entry with 16-byte cp.async copies (one TMA request per
//    four rows measured about 40 cycles each, ~2.4 us for a 96-entry tile).  The same image is
//    the K-major operand of QK (rows = entries) and the MN-major operand of PV (rows = dims).
//  - Warp 4 issues the MMAs (one thread):
//      S[entry][hi|lo head] = K_nope . [Qhi;Qlo]^T    kind::f8f6f4, E4M3 x E4M3, N = 32
//                           + K_rope . Qrope^T         kind::f16, bf16 (into the hi columns)
//      O^T[dim][hi|lo head] += V_nope^T . [Phi;Plo]^T  kind::mxf8f6f4, P scaled per 32 entries
//      O^T_rope[dim][head]  += V_rope^T . Pbf^T        kind::f16, bf16 x bf16
//    The bf16 query of each head is scaled by a power of two and split into two E4M3 terms
//    (hi = E4M3(q), lo = E4M3(q - hi)); P is split the same way after a power-of-two scale
//    per 32-entry block (the MMA's UE8M0 block scale), so each product keeps about as many
//    significant bits as a bf16 operand.  The hi and lo rows are stacked into one N = 32
//    operand and their results added when read back.  Block 3 holds bytes 384..511 (box copies;
//    a gathered tile fills only 384..447), whose upper half is the bf16 RoPE part: QK reads
//    only its first 64 bytes, and the PV rows of dims 448..511 it yields are discarded.  S and O
//    accumulate in fp32 in tensor memory.
//  - Warps 8-15 run the online softmax: thread = entry (TMEM lane); warps 8-11 own heads 0-7,
//    warps 12-15 heads 8-15.  The running max is raised lazily: O is rescaled in tensor memory
//    only when a tile's max exceeds it by more than 8 (log2 units), so P <= 256 always.  After a
//    split's first tile, P is first formed against the running max and the softmax warps meet
//    once (P published, and whether any entry lay more than 8 above the max); only then does a
//    tile take the full path: the tile maxima, the new max, O rescaled where needed, P formed
//    again (three barriers, two more when O is rescaled).  A split of one tile runs the full
//    path directly (the kernel is compiled both ways).
//  - Warps 8-15 prepare the query operands (one load per thread, issued right after the
//    upstream wait) while the first copies are in flight.
//  Three tile buffers, two S slots and two P buffers overlap the copies of tiles t+1 and t+2,
//  QK of t+1, softmax of t and PV of t-1.  Every wait is bounded.  Each split writes its
//  unnormalised O, the running max m (log2 units) and the sum l; attention_merge_kernel combines
//  the splits.
#include <stdint.h>

#include "csld_internal.cuh"
#include "kernels.cuh"
#include "sm100.cuh"

namespace csld {

namespace {

// 16 warps: copies 0-3, MMA issue 4 (warps 5-7 only take part in the start-up barrier),
// softmax 8-15
constexpr int kTcThreads = 512;
constexpr int kCopyThreads = 128;
constexpr int kMmaWarp = 4;
constexpr int kTcTile = 96;                   // entries per tile: K of PV, valid rows of QK (a multiple of 32)
constexpr int kTcRows = 128;                  // rows of the QK MMA (M); rows past kTcTile are read, never used
static_assert(kCopyThreads >= kTcTile, "each copy thread resolves at most one entry's source row");
constexpr int kBufs = 3;                      // tile buffers: copies run up to two tiles ahead of PV
constexpr int kKBlocks = kTcTile / 32;        // 32-entry K blocks of PV per tile (one P block scale each)
constexpr int kBlk = 5;                       // 128-byte column blocks per entry
constexpr int kBlkBytes = kTcTile * 128;      // 12 KB: one column block of a tile
constexpr int kTileBytes = kBlk * kBlkBytes;  // 60 KB
constexpr int kRopeBlk = 4;                   // block 4 = entry bytes 448..575 (bf16 RoPE)
constexpr uint32_t kTmemCols = 256;
// tensor-memory columns
constexpr uint32_t kColS = 0;                 // S slots at 0 and 32: hi heads +0..15, lo heads +16..31
constexpr uint32_t kColO = 64;                // O^T nope blocks at 64, 96, 128, 160 (hi +0..15, lo +16..31)
constexpr uint32_t kColOR = 192;              // O^T RoPE block 192..207
constexpr uint32_t kColSFA = 208;             // 208..211: unit scale factors of V
constexpr uint32_t kColSFB = 212;             // 212 and 216: P block scales of the two P buffers
constexpr float kRescaleLog2 = 8.f;           // lazy rescale threshold (P <= 2^8)
constexpr uint32_t kIdQK = idesc_e4m3_m128(32, false, false);
constexpr uint32_t kIdQKr = idesc_bf16_m128(16, false, false);
constexpr uint32_t kIdPVr = idesc_bf16_m128(16, true, false);
constexpr int kSmBar = 1;                     // named barrier of the 8 softmax warps (256 threads)
constexpr int kReadyBar = 2;                  // warps 4-15: query and tensor memory ready (384 threads)
constexpr int kCopyBar = 4;                   // warps 0-3: the copy warps (128 threads)

struct TcAttnSmem {
    uint8_t tile[kBufs][kTileBytes];          // [block][entry][128 B], 128-byte swizzle
    uint8_t tile_pad[(kTcRows - kTcTile) * 128];   // the QK rows read past the last block
    uint8_t qk[4][32 * 128];                  // QK B operand per nope block: rows 0..15 Qhi, 16..31 Qlo
    uint8_t qr[16 * 128];                     // RoPE query, bf16, 16 rows
    uint8_t p8[2][32 * 128];                  // PV B operand: rows 0..15 Phi, 16..31 Plo, K = 128 entries
    uint8_t pbf[2][2][16 * 128];              // bf16 P: two 64-entry K blocks of 16 rows
    float c2[kHeads];                         // log2-domain logit factor per head
    float sq[kHeads];                         // power-of-two query scale per head
    alignas(16) float tmax[2][4][kHeads];     // tile maxima per lane quarter, two sets by tile parity
    uint32_t sfb[2][4][kHeads];               // P block-scale bytes [buffer][32-entry block][head]
    float lred[4][kHeads];
    const uint8_t* src[kTcTile];              // per-entry source of the tile being gathered (null: zeros)
    uint64_t full[kBufs], empty[kBufs], sfull[2], sfree[2], pfull[2], pdone[2], drain;
    uint32_t tmem_base;
    int32_t fail, n_issued, n_landed;
};

// Non-blocking test of an mbarrier phase (the MMA issuer polls several barriers in turn; a
// try_wait could suspend it on one that is not ready while another is).
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ float order_key_to_float(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}
// 2^e as a float, -126 <= e <= 127.
__device__ __forceinline__ float pow2f(int e) { return __uint_as_float(static_cast<uint32_t>(e + 127) << 23); }

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        :: "r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar)) : "memory");
}
// 16-byte copy global -> shared through L2 (cp.async.cg); src_bytes = 0 writes 16 zero bytes and
// reads nothing.
__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
// Scales 8 consecutive TMEM columns of this warp's lanes by f[0..7].
__device__ __forceinline__ void tmem_scale8(uint32_t taddr, const float (&f)[8]) {
    uint32_t o[8];
    tmem_ld_32x32b_x8(taddr, o);
    tmem_ld_wait();
#pragma unroll
    for (int h = 0; h < 8; ++h) o[h] = __float_as_uint(__uint_as_float(o[h]) * f[h]);
    tmem_st_32x32b_x8(taddr, o);
}

// The query of head h, t = 0..255 (head t / 16, dims 32 (t % 16) .. +31), loaded once into
// registers.
__device__ __forceinline__ void qprep_load(uint4 (&v)[4], const uint16_t* q, int b, int t) {
    const uint4* src = reinterpret_cast<const uint4*>(q + ((size_t)b * kHeads + (t >> 4)) * kDim + 32 * (t & 15));
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = __ldg(src + i);
}
// Query operands from those registers.  Head h is scaled by sq = 2^(7 - floor(log2 max|q_h|)),
// so it stays below 256 (E4M3 max 448); the 16 threads of a head find max|q_h| by shuffles.
// Nope dims -> E4M3 hi and lo terms (rows h and 16 + h of the swizzled QK operand), RoPE dims
// -> bf16; each thread writes whole 16-byte chunks.
// kv_scale: the entries' FP8 dims stand for kv_scale times their code value (scaled FP8 entries;
// 1 for the base layout), so the query's FP8 part is multiplied by it before it is split (the
// output's FP8 dims are multiplied by it in the merge).
__device__ __forceinline__ void qprep_store(TcAttnSmem& sm, const uint4 (&v)[4], int t, float scale, float kv_scale) {
    const int h = t >> 4, part = t & 15, d0 = 32 * part;
    uint32_t w[16];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        w[4 * i] = v[i].x;
        w[4 * i + 1] = v[i].y;
        w[4 * i + 2] = v[i].z;
        w[4 * i + 3] = v[i].w;
    }
    float amax = 0.f;
#pragma unroll
    for (int c = 0; c < 16; ++c)
        amax = fmaxf(amax, fmaxf(fabsf(bf16_bits_to_f32(w[c] & 0xFFFFu)), fabsf(bf16_bits_to_f32(w[c] >> 16))));
    if (d0 < kNope) amax *= kv_scale;
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const int sh = amax > 0.f ? max(-100, min(100, 7 - ilogbf(amax))) : 0;
    const float sq = ldexpf(1.f, sh);
    if (part == 0) {
        sm.sq[h] = sq;
        sm.c2[h] = scale * 1.4426950408889634f / sq;
    }
    if (d0 < kNope) {
        const float sqn = sq * kv_scale;
        uint32_t hw[8], lw[8];   // bytes of dims d0 + 4c .. +3
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            uint32_t hi2[2], lo2[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const uint32_t x = w[2 * c + u];
                const float x0 = bf16_bits_to_f32(x & 0xFFFFu) * sqn, x1 = bf16_bits_to_f32(x >> 16) * sqn;
                hi2[u] = __nv_cvt_float2_to_fp8x2(make_float2(x0, x1), __NV_SATFINITE, __NV_E4M3);
                const uint32_t back = e4m3x2_to_f16x2(hi2[u]);   // exact
                const float r0 = x0 - __half2float(__ushort_as_half(static_cast<unsigned short>(back & 0xFFFFu)));
                const float r1 = x1 - __half2float(__ushort_as_half(static_cast<unsigned short>(back >> 16)));
                lo2[u] = __nv_cvt_float2_to_fp8x2(make_float2(r0, r1), __NV_SATFINITE, __NV_E4M3);
            }
            hw[c] = (hi2[0] & 0xFFFFu) | (hi2[1] << 16);
            lw[c] = (lo2[0] & 0xFFFFu) | (lo2[1] << 16);
        }
        uint8_t* blk = sm.qk[d0 >> 7];
        const int c0 = d0 & 127;
        *reinterpret_cast<uint4*>(blk + sw128(h, c0)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        *reinterpret_cast<uint4*>(blk + sw128(h, c0 + 16)) = make_uint4(hw[4], hw[5], hw[6], hw[7]);
        *reinterpret_cast<uint4*>(blk + sw128(16 + h, c0)) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
        *reinterpret_cast<uint4*>(blk + sw128(16 + h, c0 + 16)) = make_uint4(lw[4], lw[5], lw[6], lw[7]);
    } else {
        const int r0 = d0 - kNope;   // RoPE dims r0 .. r0 + 31: 64 bytes of row h
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            uint32_t o[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const uint32_t x = w[4 * j + c];
                o[c] = f32_to_bf16_bits(bf16_bits_to_f32(x & 0xFFFFu) * sq) |
                       (f32_to_bf16_bits(bf16_bits_to_f32(x >> 16) * sq) << 16);
            }
            *reinterpret_cast<uint4*>(sm.qr + sw128(h, 2 * r0 + 16 * j)) = make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
    fence_proxy_async_smem();
}

// P of one tile for this thread's entry e and its head group's 8 heads against the maxima m
// (log2 units): p = 2^(x - m), 0 for a head that has seen no visible entry yet (m = -inf).  P is
// stored as two E4M3 terms after a power-of-two scale per (32-entry block = this lane quarter,
// head) in the PV operand rows h and 16 + h, and as bf16 for the RoPE dims; the block scales go
// to sfb[head].  Heads go in pairs through the paired converts.  The p of each head goes to
// l: added (kAdd) or stored.
template <bool kAdd>
__device__ __forceinline__ void write_p(uint8_t* p8, uint8_t* pb, uint32_t* sfb, const float (&m)[8],
                                       const float (&x)[8], float (&l)[8], int hg, int e, int lane) {
#pragma unroll
    for (int h = 0; h < 8; h += 2) {
        const int hh = 8 * hg + h;
        const float p0 = m[h] == -INFINITY ? 0.f : exp2_ftz(x[h] - m[h]);
        const float p1 = m[h + 1] == -INFINITY ? 0.f : exp2_ftz(x[h + 1] - m[h + 1]);
        l[h] = kAdd ? l[h] + p0 : p0;
        l[h + 1] = kAdd ? l[h + 1] + p1 : p1;
        const uint32_t pm0 = __reduce_max_sync(0xffffffffu, __float_as_uint(p0));   // p >= 0
        const uint32_t pm1 = __reduce_max_sync(0xffffffffu, __float_as_uint(p1));
        // ks = 7 - floor(log2 max p): the scaled block stays below 256
        const int ks0 = pm0 >= 0x00800000u ? max(-126, min(127, 134 - static_cast<int>(pm0 >> 23))) : 0;
        const int ks1 = pm1 >= 0x00800000u ? max(-126, min(127, 134 - static_cast<int>(pm1 >> 23))) : 0;
        const float xs0 = p0 * pow2f(ks0), xs1 = p1 * pow2f(ks1);
        const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(xs0, xs1), __NV_SATFINITE, __NV_E4M3);
        const uint32_t back = e4m3x2_to_f16x2(hi);   // exact
        const float r0 = xs0 - __half2float(__ushort_as_half(static_cast<unsigned short>(back & 0xFFFFu)));
        const float r1 = xs1 - __half2float(__ushort_as_half(static_cast<unsigned short>(back >> 16)));
        const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(r0, r1), __NV_SATFINITE, __NV_E4M3);
        const uint32_t pbf2 = f32x2_to_bf16x2_bits(p0, p1);
        p8[sw128(hh, e)] = static_cast<uint8_t>(hi);
        p8[sw128(hh + 1, e)] = static_cast<uint8_t>(hi >> 8);
        p8[sw128(16 + hh, e)] = static_cast<uint8_t>(lo);
        p8[sw128(17 + hh, e)] = static_cast<uint8_t>(lo >> 8);
        *reinterpret_cast<uint16_t*>(pb + sw128(hh, 2 * (e & 63))) = static_cast<uint16_t>(pbf2);
        *reinterpret_cast<uint16_t*>(pb + sw128(hh + 1, 2 * (e & 63))) = static_cast<uint16_t>(pbf2 >> 16);
        if (lane == h) sfb[hh] = static_cast<uint32_t>(127 - ks0);
        if (lane == h + 1) sfb[hh + 1] = static_cast<uint32_t>(127 - ks1);
    }
}

}  // namespace

// kFast: tiles after a split's first try P against the running max first (worth it when splits
// hold several tiles; a one-tile split runs the plain path).
template <bool kFast>
__global__ void __launch_bounds__(kTcThreads, 1) attention_tc_partial_kernel(
    const __grid_constant__ CUtensorMap kv_tile, const __grid_constant__ CUtensorMap win_tile,
    const uint8_t* __restrict__ comp_kv, const uint8_t* __restrict__ win_kv,
    const uint16_t* __restrict__ q, int64_t cap, int ratio,
    const int32_t* __restrict__ topk, int k, int W, int Wr, int Q, const int32_t* __restrict__ seq_len, float scale,
    int splits, float* __restrict__ opart, float2* __restrict__ mlpart, int32_t* err, float kv_scale) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    TcAttnSmem& sm = *reinterpret_cast<TcAttnSmem*>(smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023));
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // query row vq = cache row b times Q + the query's place jq among the Q newest tokens
    const int vq = blockIdx.y, split = blockIdx.x;
    const int b = vq / Q, jq = vq % Q;

    // ---- setup --------------------------------------------------------------------------------
    if (tid == 0) {
        for (int s = 0; s < kBufs; ++s) {
            mbar_init(&sm.full[s], kCopyThreads);   // one arrival per copy thread
            mbar_init(&sm.empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&sm.sfull[s], 1);
            mbar_init(&sm.sfree[s], 8);
            mbar_init(&sm.pfull[s], 8);
            mbar_init(&sm.pdone[s], 1);
        }
        mbar_init(&sm.drain, 1);
        sm.fail = 0;
        sm.n_issued = 0;
        sm.n_landed = 0;
        fence_barrier_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(&sm.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_map(&kv_tile);
        tma_prefetch_map(&win_tile);
    }
    tc_fence_before();
    __syncthreads();   // barriers initialised, tensor memory allocated
    tc_fence_after();
    pdl_wait();      // lengths, top-k indices and the caches come from upstream
    pdl_trigger();
    uint4 qv[4];     // the softmax warps' query values, in flight while the length loads
    if (warp >= 8) qprep_load(qv, q, vq, tid - 256);

    // ---- the key list of sequence b and this split's tile range ----------------------------
    // list = [compressed slots padded to a multiple of 4 with empty slots][window tokens], so a
    // group of 4 slots never mixes the two sources
    int32_t n = seq_len[b];
    if (n < 0) {
        if (tid == 0 && split == 0) dev_error(err, CSLD_DEVERR_SEQ_LEN);
        n = 0;
    }
    n = max(0, n - (Q - 1 - jq));   // the tokens this query sees (itself included)
    const int64_t n_vis = min64(n / ratio, cap);
    const bool sparse = topk != nullptr;
    const int64_t n_comp = sparse ? (int64_t)k : n_vis;
    const int64_t n_comp4 = (n_comp + 3) & ~int64_t(3);
    const int n_win = W > 0 ? min(W, n) : 0;
    const int64_t L = n_comp4 + n_win;
    const int64_t n_tiles_all = (L + kTcTile - 1) / kTcTile;
    const int64_t t_begin = n_tiles_all * split / splits;
    const int n_tiles = static_cast<int>(n_tiles_all * (split + 1) / splits - t_begin);
    const size_t part = (size_t)vq * splits + split;
    // compressed slot i -> row of the compressed map, or -1 for an empty slot; sel = the slot's
    // top-k entry (sparse lists; loaded by sel_of, so several loads can be in flight at once)
    auto sel_of = [&](int64_t i) -> int32_t { return (sparse && i < n_comp) ? __ldg(topk + (size_t)vq * k + i) : 0; };
    auto comp_row = [&](int64_t i, int32_t sel, bool report) -> int32_t {
        if (i >= n_comp) return -1;
        int64_t v = i;
        if (sparse) {
            v = sel;
            if (v >= n_vis) {
                if (report) dev_error(err, CSLD_DEVERR_BAD_INDEX);
                return -1;
            }
            if (v < 0) return -1;
        }
        return static_cast<int32_t>((int64_t)b * cap + v);
    };

    const uint32_t tmem = sm.tmem_base;
    volatile int32_t* fail = &sm.fail;

    if (n_tiles <= 0) {
        if (tid < kHeads) mlpart[part * kHeads + tid] = make_float2(-INFINITY, 0.f);
    } else if (warp < 4) {
        // ===== copies (warps 0-3): tile t into buffer t % kBufs, started before the query is ready =====
        // Whole tiles of consecutive compressed entries (or the full window ring) come as TMA
        // boxes, one per column block.  Every other tile (selected entries, the tail, the window)
        // is gathered with 16-byte cp.async copies: entry e's 36 chunks go to row e of the five
        // column blocks (bytes 0..447 to blocks 0-3, bytes 448..575 to block 4), so a copy
        // thread moves 27 chunks and the four warps fetch whole entries in order.  A gathered
        // tile is published (fence to the async proxy, arrival on its full barrier) once the
        // thread's copies of it have landed, checked after the next tile's copies are issued.
        int t = 0, pend = -1;   // pend: the gathered tile whose arrivals are still owed
        auto publish = [&](int wait_all) {
            if (pend < 0) return;
            if (wait_all) cp_async_wait<0>();
            else cp_async_wait<1>();
            fence_proxy_async_smem();
            mbar_arrive(&sm.full[pend % kBufs]);
            pend = -1;
        };
        for (; t < n_tiles; ++t) {
            const int s = t % kBufs;
            const int64_t i0 = (t_begin + t) * kTcTile;
            uint8_t* tl = sm.tile[s];
            const bool box_comp = !sparse && i0 + kTcTile <= n_comp;
            // the tile is the whole window and the ring is full: its W slots hold exactly those
            // tokens (in ring order, which the softmax does not care about)
            const bool box_win = W == kTcTile && Wr == W && n_win == W && i0 == n_comp4;
            const bool ok = !*fail && (t < kBufs || mbar_wait(&sm.empty[s], ((t / kBufs) - 1) & 1));
            if (named_barrier_or(kCopyBar, kCopyThreads, !ok)) {   // the copy warps leave together
                publish(1);
                if (tid == 0) *fail = 1;
                break;
            }
            if (box_comp || box_win) {
                publish(1);
                if (tid == 0) mbar_arrive_expect_tx(&sm.full[s], kTileBytes);
                else mbar_arrive(&sm.full[s]);
                if (tid < kBlk) {
                    const int x = tid < 4 ? 128 * tid : kNope;
                    if (box_comp) tma_load_2d(tl + tid * kBlkBytes, &kv_tile, x, static_cast<int>((int64_t)b * cap + i0), &sm.full[s]);
                    else tma_load_2d(tl + tid * kBlkBytes, &win_tile, x, b * W, &sm.full[s]);
                }
                continue;
            }
            if (tid < kTcTile) {   // entry tid's source row
                const int64_t i = i0 + tid;
                const uint8_t* src = nullptr;
                if (i < n_comp4) {
                    const int32_t row = comp_row(i, sel_of(i), true);
                    if (row >= 0) src = comp_kv + (size_t)row * kEntry;
                } else if (i < L && win_kv != nullptr) {
                    const int64_t tok = (int64_t)n - n_win + (i - n_comp4);
                    src = win_kv + ((size_t)b * Wr + (size_t)(tok % Wr)) * kEntry;
                }
                sm.src[tid] = src;
            }
            named_barrier(kCopyBar, kCopyThreads);
#pragma unroll 3
            for (int g = tid; g < kTcTile * (kEntry / 16); g += kCopyThreads) {
                const int e = g / (kEntry / 16), c = g - e * (kEntry / 16);
                const uint8_t* src = sm.src[e];
                uint8_t* dst = c < 28 ? tl + (c >> 3) * kBlkBytes + sw128(e, 16 * (c & 7))
                                      : tl + kRopeBlk * kBlkBytes + sw128(e, 16 * (c - 28));
                cp_async16(dst, src ? src + 16 * c : comp_kv, src ? 16u : 0u);
            }
            cp_async_commit();
            publish(0);   // the tile before, if it was gathered
            pend = t;
        }
        publish(1);
        if (tid == 0) sm.n_issued = t;
    } else if (warp >= 4 && warp < 8) {
        // ===== warps 4-7 wait for the query operands and tensor memory (written by warps 8-15) ====
        named_barrier(kReadyBar, 384);
        tc_fence_after();
        if (warp == kMmaWarp && lane == 0) {
            // ===== MMA issue (one thread) =========================================================
            const uint64_t dq = desc_sw128(sm.qk[0], 0), dqr = desc_sw128(sm.qr, 0);
            // Issue whatever is ready, PV first (it frees a tile buffer for the next copy):
            // PV(np) once P(np) is published; QK(nq) once tile nq landed and its S slot is free.
            // The polls do not block (test_wait), so a barrier that is not ready never holds up
            // another that is.
            int nq = 0, np = 0, landed = 0;
            uint32_t idle = 0;
            while (np < n_tiles) {
                if (*fail) break;
                if (np < nq && mbar_test_wait(&sm.pfull[np & 1], (np >> 1) & 1)) {
                    const int su = np & 1, sb = np % kBufs;   // P buffer, tile buffer
                    tc_fence_after();
                    const uint64_t da = desc_sw128(sm.tile[sb], 0);
                    const uint64_t dp = desc_sw128(sm.p8[su], 0);
                    const uint32_t sfb0 = tmem + kColSFB + 4u * su;
#pragma unroll
                    for (int mb = 0; mb < 4; ++mb)
#pragma unroll
                        for (int kb = 0; kb < kKBlocks; ++kb)   // 32 entries (4 row groups) per MMA
                            umma_mxf8f6f4(tmem + kColO + 32u * mb, da + (mb * kBlkBytes + kb * 4096) / 16,
                                          dp + (32 * kb) / 16, idesc_mxe4m3_m128(32, true, false, kb), tmem + kColSFA,
                                          sfb0 | (static_cast<uint32_t>(kb) << 30), 1u);
                    // RoPE: M = 128 with LBO one block (rows 64..127 read the next block: unused)
                    const uint64_t dar = desc_sw128(sm.tile[sb] + kRopeBlk * kBlkBytes, kBlkBytes);
                    const uint64_t dpb = desc_sw128(sm.pbf[su][0], 0);
#pragma unroll
                    for (int ks = 0; ks < kTcTile / 16; ++ks)
                        umma_f16(tmem + kColOR, dar + (ks * 2048) / 16, dpb + ((ks >> 2) * 2048 + 32 * (ks & 3)) / 16,
                                 kIdPVr, 1u);
                    umma_commit(&sm.empty[sb]);
                    umma_commit(&sm.pdone[su]);
                    ++np;
                    idle = 0;
                    continue;
                }
                if (nq < n_tiles && nq < np + 2 && mbar_test_wait(&sm.full[nq % kBufs], (nq / kBufs) & 1) &&
                    (nq < 2 || mbar_test_wait(&sm.sfree[nq & 1], ((nq >> 1) - 1) & 1))) {
                    const int s = nq & 1;   // S slot
                    landed = nq + 1;
                    tc_fence_after();
                    const uint32_t dS = tmem + kColS + 32u * s;
                    const uint64_t da = desc_sw128(sm.tile[nq % kBufs], 0);
#pragma unroll
                    for (int kb = 0; kb < 4; ++kb)
#pragma unroll
                        for (int ks = 0; ks < (kb < 3 ? 4 : 2); ++ks)   // 32 bytes of K per MMA; block 3
                            // stops at byte 448 (the RoPE half is bf16: as E4M3 it may hold NaNs)
                            umma_f8f6f4(dS, da + (kb * kBlkBytes + 32 * ks) / 16, dq + (kb * 4096 + 32 * ks) / 16, kIdQK,
                                        (kb | ks) != 0 ? 1u : 0u);
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        umma_f16(dS, da + (kRopeBlk * kBlkBytes + 32 * ks) / 16, dqr + (32 * ks) / 16, kIdQKr, 1u);
                    umma_commit(&sm.sfull[s]);
                    ++nq;
                    idle = 0;
                    continue;
                }
                if (++idle > (1u << 22)) {   // nothing became ready for about a second
                    *fail = 1;
                    break;
                }
                if (idle > 64) __nanosleep(32);
            }
            sm.n_landed = landed;
        }
    } else if (warp >= 8) {
        // ===== online softmax: thread = entry e = TMEM lane; head group hg = 8 heads =============
        const int sub = warp & 3, hg = (warp - 8) >> 2, e = 32 * sub + lane;
        const uint32_t lb = tmem + ((32u * sub) << 16);
        if (hg == 0) {   // O = 0 and unit scale factors of V for this lane quarter
            for (uint32_t c = kColO; c < kColSFA; c += 8) tmem_st_32x32b_x8_fill(lb + c, 0u);
            tmem_st_32x32b_x8_fill(lb + kColSFA, 0x7F7F7F7Fu);
            tmem_st_wait();
        }
        qprep_store(sm, qv, tid - 256, scale, kv_scale);
        tc_fence_before();
        named_barrier(kReadyBar, 384);
        tc_fence_after();
        float c2[8], mref[8], lsum[8];
#pragma unroll
        for (int h = 0; h < 8; ++h) {
            c2[h] = sm.c2[8 * hg + h];
            mref[h] = -INFINITY;
            lsum[h] = 0.f;
        }
        bool ok = true;
        for (int t = 0; t < n_tiles; ++t) {
            const int s = t & 1;
            const int64_t i = (t_begin + t) * kTcTile + e;
            const bool valid = e < kTcTile && (i < n_comp4 ? comp_row(i, sel_of(i), false) >= 0 : i < L);
            ok = __all_sync(0xffffffffu, !*fail && mbar_wait(&sm.sfull[s], (t >> 1) & 1));
            float x[8];
            if (ok) {
                tc_fence_after();
                uint32_t shi[8], slo[8];
                tmem_ld_32x32b_x8(lb + kColS + 32u * s + 8u * hg, shi);
                tmem_ld_32x32b_x8(lb + kColS + 32u * s + 16u + 8u * hg, slo);
                tmem_ld_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.sfree[s]);
#pragma unroll
                for (int h = 0; h < 8; ++h)
                    x[h] = valid ? (__uint_as_float(shi[h]) + __uint_as_float(slo[h])) * c2[h] : -INFINITY;
            } else {
#pragma unroll
                for (int h = 0; h < 8; ++h) x[h] = -INFINITY;
            }
            // Fast path: no entry of this tile lies more than 2^8 above the running max (the common
            // case after a split's first tile), so P is formed against m as it stands and the
            // softmax warps meet once, where they publish P.  Otherwise (a new maximum, the first
            // tile, or a failed wait) the tile takes the full path: tile maxima, new m, O
            // rescaled, P formed again.
            bool over = true;
            if constexpr (kFast) {
                over = !ok;
#pragma unroll
                for (int h = 0; h < 8; ++h) over |= x[h] > mref[h] + kRescaleLog2;
                // P buffer s is free once PV(t-2) completed
                if (t >= 2 && !over) over = !mbar_wait(&sm.pdone[s], ((t >> 1) - 1) & 1);
            }
            // pass 0 (not on a split's first tile): P against the running max, kept when no warp
            // saw a new maximum; pass 1: the full path
            float ladd[8];
            bool quit = false, kept = false;   // kept: the P of pass 0 stands
            for (int pass = (kFast && t > 0) ? 0 : 1; pass < 2; ++pass) {
                if (pass == 1) {
                    // tile max per head: warp max of order keys, published per lane quarter (two sets,
                    // alternating by tile, so the next tile's maxima never overwrite ones still read)
#pragma unroll
                    for (int h = 0; h < 8; ++h) {
                        const uint32_t km = __reduce_max_sync(0xffffffffu, score_key(x[h]));
                        if (lane == h) sm.tmax[s][sub][8 * hg + h] = order_key_to_float(km);
                    }
                    if (named_barrier_or(kSmBar, 256, !ok)) {   // maxima published; the warps leave together
                        quit = true;
                        break;
                    }
                    bool rescale = false;
                    float mnew[8];
                    {
                        float tm[8];
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {   // the four quarters' maxima of this warp's 8 heads
                            const float4 a = *reinterpret_cast<const float4*>(&sm.tmax[s][q4][8 * hg]);
                            const float4 c = *reinterpret_cast<const float4*>(&sm.tmax[s][q4][8 * hg + 4]);
                            const float v[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
#pragma unroll
                            for (int h = 0; h < 8; ++h) tm[h] = q4 == 0 ? v[h] : fmaxf(tm[h], v[h]);
                        }
#pragma unroll
                        for (int h = 0; h < 8; ++h) {
                            mnew[h] = (tm[h] > mref[h] + kRescaleLog2 || mref[h] == -INFINITY) ? fmaxf(tm[h], mref[h]) : mref[h];
                            rescale |= (mnew[h] != mref[h]) && (mref[h] != -INFINITY);
                        }
                    }
                    // P buffer s is free once PV(t-2) completed; a rescale of O also needs PV(t-1) done
                    // (two more barriers, taken only when some head must be rescaled or a wait failed).
                    if (t >= 2) ok = mbar_wait(&sm.pdone[s], ((t >> 1) - 1) & 1);
                    if (named_barrier_or(kSmBar, 256, rescale || !ok)) {
                        if (named_barrier_or(kSmBar, 256, !ok)) {
                            quit = true;
                            break;
                        }
                        if (t >= 1) ok = mbar_wait(&sm.pdone[(t - 1) & 1], ((t - 1) >> 1) & 1);
                        if (named_barrier_or(kSmBar, 256, !ok)) {
                            quit = true;
                            break;
                        }
                    }
                    tc_fence_after();
                    if (rescale) {   // l, and this warp's 8 heads in every O block of its lane quarter
                        float f[8];
#pragma unroll
                        for (int h = 0; h < 8; ++h) {
                            f[h] = (mref[h] == -INFINITY || mref[h] == mnew[h]) ? 1.f : exp2_ftz(mref[h] - mnew[h]);
                            lsum[h] *= f[h];
                        }
#pragma unroll 1
                        for (int blk = 0; blk < 4; ++blk) {
                            tmem_scale8(lb + kColO + 32u * blk + 8u * hg, f);
                            tmem_scale8(lb + kColO + 32u * blk + 16u + 8u * hg, f);
                        }
                        tmem_scale8(lb + kColOR + 8u * hg, f);
                        tmem_st_wait();
                    }
#pragma unroll
                    for (int h = 0; h < 8; ++h) mref[h] = mnew[h];
                }
                if (pass == 1)
                    write_p<true>(sm.p8[s], sm.pbf[s][e >> 6], sm.sfb[s][sub], mref, x, lsum, hg, e, lane);
                else if (kFast && !__any_sync(0xffffffffu, over))
                    write_p<false>(sm.p8[s], sm.pbf[s][e >> 6], sm.sfb[s][sub], mref, x, ladd, hg, e, lane);
                fence_proxy_async_smem();
                // P published; after pass 0 the warps also learn whether any saw a new maximum
                if (!kFast) {
                    named_barrier(kSmBar, 256);
                    break;
                }
                if (!named_barrier_or(kSmBar, 256, pass == 0 && over)) {
                    kept = pass == 0;
                    break;
                }
            }
            if (quit) {
                ok = false;
                break;
            }
            if (kFast && kept) {
#pragma unroll
                for (int h = 0; h < 8; ++h) lsum[h] += ladd[h];
            }
            if (hg == 0) {   // block-scale word of row `lane` (rows h and 16 + h: head lane & 15)
                const int hh = lane & 15;
                const uint32_t wsf = sm.sfb[s][0][hh] | (sm.sfb[s][1][hh] << 8) | (sm.sfb[s][2][hh] << 16) |
                                     (sm.sfb[s][3][hh] << 24);
                tmem_st_32x32b_x1(lb + kColSFB + 4u * s, wsf);
                tmem_st_wait();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.pfull[s]);
        }
        // ---- the split's results ---------------------------------------------------------
        if (ok) {
            const int tl = n_tiles - 1;
            ok = !named_barrier_or(kSmBar, 256, !mbar_wait(&sm.pdone[tl & 1], (tl >> 1) & 1));
        }
        if (ok) {
            tc_fence_after();
            float* ob = opart + part * kHeads * kDim;
#pragma unroll 1
            for (int blk = 0; blk < 4; ++blk) {
                uint32_t oh[8], ol[8];
                tmem_ld_32x32b_x8(lb + kColO + 32u * blk + 8u * hg, oh);
                tmem_ld_32x32b_x8(lb + kColO + 32u * blk + 16u + 8u * hg, ol);
                tmem_ld_wait();
                const int d = 128 * blk + e;
                if (d < kNope) {
#pragma unroll
                    for (int h = 0; h < 8; ++h) ob[(8 * hg + h) * kDim + d] = __uint_as_float(oh[h]) + __uint_as_float(ol[h]);
                }
            }
            {
                uint32_t o[8];
                tmem_ld_32x32b_x8(lb + kColOR + 8u * hg, o);
                tmem_ld_wait();
                if (e < kRope) {
#pragma unroll
                    for (int h = 0; h < 8; ++h) ob[(8 * hg + h) * kDim + kNope + e] = __uint_as_float(o[h]);
                }
            }
#pragma unroll
            for (int h = 0; h < 8; ++h) {
                float v = lsum[h];
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
                if (lane == h) sm.lred[sub][8 * hg + h] = v;
            }
            named_barrier(kSmBar, 256);
            if (sub == 0 && lane < 8) {
                float mine = -INFINITY;
#pragma unroll
                for (int h = 0; h < 8; ++h) mine = (lane == h) ? mref[h] : mine;
                const int hh = 8 * hg + lane;
                mlpart[part * kHeads + hh] =
                    make_float2(mine, (sm.lred[0][hh] + sm.lred[1][hh]) + (sm.lred[2][hh] + sm.lred[3][hh]));
            }
        } else {
            *fail = 1;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (sm.fail) {
        // a bounded wait gave up: record it, let the copies and MMAs in flight finish (bounded),
        // publish nothing
        if (warp == kMmaWarp && lane == 0) {
            dev_error(err, CSLD_DEVERR_TIMEOUT);
            for (int t = sm.n_landed; t < sm.n_issued; ++t) (void)mbar_wait(&sm.full[t % kBufs], (t / kBufs) & 1);
            umma_commit(&sm.drain);
            (void)mbar_wait(&sm.drain, 0);
        }
        if (tid < kHeads) mlpart[part * kHeads + tid] = make_float2(-INFINITY, 0.f);
        __syncthreads();
    }
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

size_t attention_tc_smem_bytes() { return sizeof(TcAttnSmem) + 1024; }
int attention_tc_tile() { return kTcTile; }

cudaError_t launch_attention_tc_partial(const uint16_t* q, const uint8_t* comp_kv, int64_t cap, int ratio,
                                        const int32_t* topk, int k, const uint8_t* win_kv, int W, int Wr, int Q,
                                        const int32_t* seq_len, int B, float scale, int splits, float* opart,
                                        float2* mlpart, int32_t* err, cudaStream_t stream, float kv_scale) {
    // the caches as 2-D byte tensors [rows][576] for the box copies of whole tiles: 128-byte
    // boxes with the 128-byte swizzle, kTcTile rows tall.  B cache rows, each serving Q query
    // rows; the window ring has Wr >= W slots per cache row.  Gathered tiles read the caches
    // through the plain pointers.
    CUtensorMap kv_tile, win_tile;
    const uint64_t rows = (uint64_t)B * (uint64_t)cap;
    if (!make_tensor_map_2d_u8(&kv_tile, comp_kv, kEntry, rows, 128, kTcTile)) return cudaErrorInvalidValue;
    const bool has_win = W > 0 && win_kv != nullptr;
    // the gathers copy 16-byte chunks of 576-byte entries
    if ((reinterpret_cast<uintptr_t>(comp_kv) & 15) != 0 || (has_win && (reinterpret_cast<uintptr_t>(win_kv) & 15) != 0))
        return cudaErrorInvalidValue;
    // a full ring of kTcTile slots as one tile (only used when W == Wr == kTcTile)
    const bool win_box = has_win && W == kTcTile && Wr == W;
    if (!make_tensor_map_2d_u8(&win_tile, win_box ? win_kv : comp_kv, kEntry, win_box ? (uint64_t)B * W : rows, 128,
                               win_box ? kTcTile : 1))
        return cudaErrorInvalidValue;
    const size_t smem = attention_tc_smem_bytes();
    // splits of more than one tile take the first-try path (the longest list: k or cap entries,
    // padded to a multiple of 4, plus the window)
    const int64_t l_max = (((topk ? (int64_t)k : cap) + 3) & ~int64_t(3)) + W;
    const int64_t tiles_per_split = ((l_max + kTcTile - 1) / kTcTile + splits - 1) / splits;
    auto kernel = tiles_per_split > 1 ? attention_tc_partial_kernel<true> : attention_tc_partial_kernel<false>;
    cudaError_t e = set_smem_once(kernel, smem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(kernel, dim3(splits, B * Q), dim3(kTcThreads), smem, stream, kv_tile, win_tile,
                   comp_kv, has_win ? win_kv : nullptr, q, cap, ratio, topk, k, W, Wr, Q, seq_len,
                   scale, splits, opart, mlpart, err, kv_scale);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace csld
