// Prefill compression: softmax-gated pooling with a learned positional bias into 576-byte
// FP8/bf16 entries, plus the FP4 lightning-indexer key of each CSA entry.
//
// Source: "DeepSeek-V4: a million-token context that agents can actually use" -- CSA paragraph
// and Figure 3 caption (4 tokens -> one entry by softmax-gated pooling with a positional bias;
// FP4 lightning indexer over the compressed entries), HCA paragraph and Figure 4 caption (128
// tokens -> one entry), storage paragraph (FP8 entries, bf16 RoPE dims, FP4 indexer).
//
// Layout: one warp pools one entry; lane l owns dims [16l, 16l+16).  The raw stream is read
// once with 16-byte loads (HBM-bound).  For CSA the pooled vectors of a 128-entry tile are
// staged as bf16 in shared memory and projected by W_I (512x64, bf16 copy resident in shared
// memory for the whole persistent CTA) on the 5th-generation tensor cores (tcgen05.mma
// kind::f16, fp32 accumulation in tensor memory); the FP4 quantisation runs on the fp32 result.
//
// Layout variants of the storage paragraph, compiled into the same kernels (kVar):
//  - kVarRope, RoPE at compressed positions: the raw tokens' dims 448..511 are taken before
//    rotary encoding and rotated here -- a pooled entry at its block's last token, a window
//    entry at its own token (RoFormer pairs, see rope_lane);
//  - kVarScaled, scaled FP8 entries: one scale sigma per layer cache, the FP8 dims stored as
//    E4M3(x / sigma) (the kernels get 1 / sigma), the RoPE dims and the indexer key unscaled;
//  - kVarPerHead, per-head indexer keys: W_I [512][4][64], one FP4 key per head and entry,
//    stored as 128-byte rows [head][32 code bytes] pre-swizzled for a 128-byte-swizzle K-major
//    operand (16-byte chunk c of entry s at chunk c ^ (s mod 8)), scales [entry][head][group].
#include "csld_internal.cuh"
#include "kernels.cuh"
#include "sm100.cuh"

namespace csld {

// 16-byte row load.  kReadOnly: the rows are not written by the running kernel, so the
// read-only path may be used; otherwise a plain (coherent) load.
template <bool kReadOnly>
__device__ __forceinline__ uint4 load_row16(const uint4* p) {
    if constexpr (kReadOnly) return __ldg(p);
    else return *p;
}

// Pools the m rows of one block.  rows: [m][512] bf16; gate, bias: [m].  Lane l returns the
// fp32 pooled values of dims [16l, 16l+16) in c[].  Deterministic order: weights are
// normalised by a warp-tree sum, the weighted sum runs over j = 0..m-1 with fmaf.
// Softmax weights of the m <= 128 slots of a block: lane l returns the weights of slots
// l, l+32, l+64, l+96 in w[] (0 past m).
__device__ __forceinline__ void warp_pool_weights(const float* gate, const float* __restrict__ bias, int m,
                                                  int lane, float (&w)[4]) {
    float a[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int j = lane + 32 * i;
        a[i] = (j < m) ? gate[j] + bias[j] : -INFINITY;
    }
    float mx = fmaxf(fmaxf(a[0], a[1]), fmaxf(a[2], a[3]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float e[4], s = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        e[i] = (lane + 32 * i < m) ? expf(a[i] - mx) : 0.f;
        s += e[i];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] = e[i] / s;
}

// The same weights for m <= 32 from values the caller loaded ahead: lane l < m passes
// gate[l] + bias[l] in a0.  The operations and their order are those of warp_pool_weights (its
// slots past lane 31 contribute -inf to the maximum and 0 to the sum), so the weights are
// bit-identical to it.
__device__ __forceinline__ void warp_pool_weights_pre(float a0, int m, int lane, float (&w)[4]) {
    float a[4] = {lane < m ? a0 : -INFINITY, -INFINITY, -INFINITY, -INFINITY};
    float mx = fmaxf(fmaxf(a[0], a[1]), fmaxf(a[2], a[3]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float e[4], s = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        e[i] = (lane + 32 * i < m) ? expf(a[i] - mx) : 0.f;
        s += e[i];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] = e[i] / s;
}

template <bool kReadOnly>
__device__ __forceinline__ void warp_pool(const uint16_t* rows, const float* gate,
                                          const float* __restrict__ bias, int m, int lane,
                                          float (&c)[16]) {
    float w[4];
#pragma unroll
    for (int d = 0; d < 16; ++d) c[d] = 0.f;
    const uint4* base = reinterpret_cast<const uint4*>(rows) + 2 * lane;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if (32 * i >= m) break;
        const int jn = min(32, m - 32 * i);
        // eight rows per batch: all sixteen 16-byte loads of a lane are issued before the
        // first is used, then the rows are added in order (one fmaf per row and dim)
        for (int j0 = 0; j0 < jn; j0 += 8) {
            uint4 x[8][2];
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                const int j = 32 * i + j0 + r;
                if (j0 + r < jn) {
                    x[r][0] = load_row16<kReadOnly>(base + (size_t)j * (kDim / 8));
                    x[r][1] = load_row16<kReadOnly>(base + (size_t)j * (kDim / 8) + 1);
                }
            }
            // the weights, once, while the first batch of rows is in flight
            if (i == 0 && j0 == 0) warp_pool_weights(gate, bias, m, lane, w);
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                if (j0 + r >= jn) break;
                const float wj = __shfl_sync(0xffffffffu, w[i], j0 + r);
                const uint32_t xv[8] = {x[r][0].x, x[r][0].y, x[r][0].z, x[r][0].w,
                                        x[r][1].x, x[r][1].y, x[r][1].z, x[r][1].w};
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    c[2 * q] = fmaf(wj, bf16_bits_to_f32(xv[q]), c[2 * q]);
                    c[2 * q + 1] = fmaf(wj, bf16_bits_to_f32(xv[q] >> 16), c[2 * q + 1]);
                }
            }
        }
    }
}

// RoPE of a pooled vector held by a warp (lane l: dims 16l..16l+15; lanes 28..31 hold the RoPE
// dims 448..511): pair i = dims (448 + 2i, 449 + 2i) turned by the angle pos * base^(-i/32)
// (RoFormer).  The angle, its sine and cosine and the products in double (the position may be
// in the millions), the result rounded to fp32.
__device__ __forceinline__ void rope_lane(float (&c)[16], int lane, int64_t pos, double base) {
    if (lane < kNope / 16) return;
#pragma unroll
    for (int p = 0; p < 8; ++p) {
        const int i = 8 * (lane - kNope / 16) + p;
        double sn, cs;
        sincos(static_cast<double>(pos) * pow(base, -static_cast<double>(i) / 32.0), &sn, &cs);
        const double x0 = c[2 * p], x1 = c[2 * p + 1];
        c[2 * p] = static_cast<float>(x0 * cs - x1 * sn);
        c[2 * p + 1] = static_cast<float>(x0 * sn + x1 * cs);
    }
}
// The same rotation for four consecutive RoPE dims 448 + 4j .. 448 + 4j + 3 held as bf16 (two
// pairs), rounded back to bf16: a window entry's RoPE part.
__device__ __forceinline__ uint2 rope_bf16x4(uint2 x, int j, int64_t pos, double base) {
    const float v[4] = {bf16_bits_to_f32(x.x), bf16_bits_to_f32(x.x >> 16), bf16_bits_to_f32(x.y),
                        bf16_bits_to_f32(x.y >> 16)};
    uint32_t w[2];
#pragma unroll
    for (int p = 0; p < 2; ++p) {
        double sn, cs;
        sincos(static_cast<double>(pos) * pow(base, -static_cast<double>(2 * j + p) / 32.0), &sn, &cs);
        const double x0 = v[2 * p], x1 = v[2 * p + 1];
        w[p] = f32_to_bf16_bits(static_cast<float>(x0 * cs - x1 * sn)) |
               (f32_to_bf16_bits(static_cast<float>(x0 * sn + x1 * cs)) << 16);
    }
    return make_uint2(w[0], w[1]);
}

constexpr int kVarBase = 0, kVarRope = 1, kVarScaled = 2, kVarPerHead = 3;
constexpr int kIkeyHead = kIdxHeads * kIkey;   // 128 bytes of per-head key codes per entry

// FP4 codes (4 words = 16 bytes) and the power-of-two scale of one 32-element group of fp32
// values u[0..1][0..15] (the same quantisation as the shared key).
__device__ __forceinline__ void fp4_group_words(const uint32_t (&u)[2][16], float* sc, uint32_t (&words)[4]) {
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(__uint_as_float(u[i >> 4][i & 15])));
    *sc = fp4_group_scale(amax);
    const float inv = 1.0f / *sc;   // exact: a power of two
#pragma unroll
    for (int wq = 0; wq < 4; ++wq) {
        uint32_t word = 0u;
#pragma unroll
        for (int bq = 0; bq < 4; ++bq) {
            const int i = 8 * wq + 2 * bq;
            const uint32_t byte = e2m1_code(__uint_as_float(u[i >> 4][i & 15]) * inv) |
                                  (e2m1_code(__uint_as_float(u[(i + 1) >> 4][(i + 1) & 15]) * inv) << 4);
            word |= byte << (8 * bq);
        }
        words[wq] = word;
    }
}

// E4M3 codes of four consecutive FP8 dims of a raw token held as bf16 (a window entry's FP8
// part); kScaled: times inv_scale first.
template <bool kScaled>
__device__ __forceinline__ uint32_t fp8x4_of_bf16x4(uint2 x, float inv_scale) {
    float v[4] = {bf16_bits_to_f32(x.x), bf16_bits_to_f32(x.x >> 16), bf16_bits_to_f32(x.y), bf16_bits_to_f32(x.y >> 16)};
    if constexpr (kScaled) {
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] *= inv_scale;
    }
    return f32_to_e4m3(v[0]) | (f32_to_e4m3(v[1]) << 8) | (f32_to_e4m3(v[2]) << 16) | (f32_to_e4m3(v[3]) << 24);
}

// Writes the 576-byte entry of the pooled vector held by the warp (lane l: dims 16l..16l+15);
// kScaled: the FP8 dims times inv_scale (= 1 / sigma) before rounding.
template <bool kScaled = false>
__device__ __forceinline__ void warp_store_entry(uint8_t* __restrict__ entry, int lane,
                                                 const float (&c)[16], float inv_scale = 1.f) {
    if (lane < kNope / 16) {
        float v[16];
#pragma unroll
        for (int d = 0; d < 16; ++d) v[d] = kScaled ? c[d] * inv_scale : c[d];
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
            w[q] = f32_to_e4m3(v[4 * q]) | (f32_to_e4m3(v[4 * q + 1]) << 8) |
                   (f32_to_e4m3(v[4 * q + 2]) << 16) | (f32_to_e4m3(v[4 * q + 3]) << 24);
        *reinterpret_cast<uint4*>(entry + 16 * lane) = make_uint4(w[0], w[1], w[2], w[3]);
    } else {
        uint32_t w[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) w[q] = f32_to_bf16_bits(c[2 * q]) | (f32_to_bf16_bits(c[2 * q + 1]) << 16);
        uint4* dst = reinterpret_cast<uint4*>(entry + kNope + 32 * (lane - kNope / 16));
        dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
        dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
    }
}

// FP4-quantises the 64-vector u (lane l holds u[2l], u[2l+1]) into 32 code bytes + 2 scales.
// Entry s's code bytes go to their stored positions: the two 16-byte halves (the two
// 32-element groups) are swapped when bit 2 of s is set (the key cache layout of csld.h).
__device__ __forceinline__ void warp_store_fp4(uint8_t* __restrict__ codes, float* __restrict__ scales,
                                               int64_t s, int lane, float u0, float u1) {
    float amax = fmaxf(fabsf(u0), fabsf(u1));
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float sg = fp4_group_scale(amax);    // lanes 0..15: group 0, lanes 16..31: group 1
    const float inv = 1.0f / sg;               // exact: sg is a power of two
    const uint32_t byte = e2m1_code(u0 * inv) | (e2m1_code(u1 * inv) << 4);
    codes[lane ^ (static_cast<int>((s >> 2) & 1) << 4)] = static_cast<uint8_t>(byte);
    if ((lane & 15) == 0) scales[lane >> 4] = sg;
}

// Per-head keys: head h's FP4 key of entry s (lane l holds u[2l], u[2l+1] of the head's 64-vector)
// into the entry's 128-byte row (chunk 2h + g at chunk (2h + g) ^ (s mod 8)) and its two scales
// into scales[2h], scales[2h + 1].
__device__ __forceinline__ void warp_store_fp4_head(uint8_t* __restrict__ row, float* __restrict__ scales, int64_t s,
                                                    int h, int lane, float u0, float u1) {
    float amax = fmaxf(fabsf(u0), fabsf(u1));
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float sg = fp4_group_scale(amax);    // lanes 0..15: group 0, lanes 16..31: group 1
    const float inv = 1.0f / sg;               // exact: sg is a power of two
    const uint32_t byte = e2m1_code(u0 * inv) | (e2m1_code(u1 * inv) << 4);
    const int g = lane >> 4;
    row[16 * ((2 * h + g) ^ static_cast<int>(s & 7)) + (lane & 15)] = static_cast<uint8_t>(byte);
    if ((lane & 15) == 0) scales[2 * h + g] = sg;
}

// ------------------------------------------------------------------------------------------
// Pooling without an indexer key (HCA, or any ratio).  One warp per entry.
// ------------------------------------------------------------------------------------------
template <int kVar>
__global__ void __launch_bounds__(256) pool_kernel(const uint16_t* __restrict__ raw,
                                                   const float* __restrict__ gate,
                                                   const float* __restrict__ bias, int m,
                                                   int64_t T, int64_t E, int B,
                                                   int64_t out_seq_stride,
                                                   uint8_t* __restrict__ kv_out, int64_t pos0, double rope_base,
                                                   float inv_scale) {
    const int lane = threadIdx.x & 31;
    const int64_t gw = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (gw >= E * B) return;
    const int64_t b = gw / E, s = gw % E;
    float c[16];
    warp_pool<true>(raw + ((size_t)b * T + (size_t)s * m) * kDim, gate + (size_t)b * T + (size_t)s * m,
              bias, m, lane, c);
    if constexpr (kVar == kVarRope) rope_lane(c, lane, pos0 + (s + 1) * m - 1, rope_base);
    warp_store_entry<kVar == kVarScaled>(kv_out + ((size_t)b * out_seq_stride + (size_t)s) * kEntry, lane, c, inv_scale);
}

// ------------------------------------------------------------------------------------------
// Pooling + indexer key (CSA) on the 5th-generation tensor cores.  Persistent CTAs (one per
// SM) of 16 warps, each over an even share of the entries in tiles of up to 128 entries:
//  1. every warp pools 8 entries of the tile (one warp per entry, as above; for m = 4 two
//     entries' raw rows are loaded at once, 256 bytes per lane in flight) and writes each
//     entry to the cache and its bf16 copy into shared memory as row r of the A operand
//     ([128 entries][512 dims], K-major, 128-byte swizzle: 8 column blocks of 64 dims);
//  2. one thread issues the projection U = A . W_I (tcgen05.mma kind::f16, M = 128 entries,
//     N = 64, K = 512 in 32 steps of 16; W_I^T resident in shared memory in the same layout)
//     into 64 fp32 columns of tensor memory;
//  3. warps 0-7 read U back (thread = entry = TMEM lane; warps 0-3 the first 32-value group,
//     warps 4-7 the second) and FP4-quantise it in registers, writing 16 code bytes (stored
//     layout of csld.h) and a scale each.
// Each warp's first write of the next tile's A rows waits for the MMA that read the previous
// tile, so the pooling loads of the next tile are already in flight meanwhile.
// ------------------------------------------------------------------------------------------
constexpr int kCTile = 128;                // entries per tile = the MMA's M
constexpr int kCThreads = 512;
constexpr int kRif = 2;                    // rows (entries) a warp has loaded at once
constexpr uint32_t kCTmemCols = 64;        // U: 128 lanes x 64 fp32 columns
constexpr uint32_t kIdProj = idesc_bf16_m128(kIdxDim, false, false);

struct CompressSmem {
    uint8_t a[kDim / 64][kCTile * 128];    // pooled rows, bf16: column block kb holds dims 64kb..64kb+63
    uint8_t w[kDim / 64][kIdxDim * 128];   // W_I^T, bf16: row n of block kb holds W_I[64kb..64kb+63][n]
    uint64_t mma_done;
    uint32_t tmem_base;
    int32_t fail;
};

// The 4 raw rows of an m = 4 block, this lane's 16 dims: x[2j], x[2j+1] = token j.
__device__ __forceinline__ void load_block4(const uint16_t* rows, int lane, uint4 (&x)[8]) {
    const uint4* base = reinterpret_cast<const uint4*>(rows) + 2 * lane;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        x[2 * j] = __ldg(base + (size_t)j * (kDim / 8));
        x[2 * j + 1] = __ldg(base + (size_t)j * (kDim / 8) + 1);
    }
}
// Weighted sum of preloaded m = 4 rows, in the order warp_pool uses (slot 0, 1, 2, 3, one fmaf
// per slot and dim), so the pooled values are bit-identical to it.
__device__ __forceinline__ void pool4_preloaded(const uint4 (&x)[8], const float (&w)[4], float (&c)[16]) {
#pragma unroll
    for (int d = 0; d < 16; ++d) c[d] = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float wj = __shfl_sync(0xffffffffu, w[0], j);
        const uint32_t xv[8] = {x[2 * j].x, x[2 * j].y, x[2 * j].z, x[2 * j].w,
                                x[2 * j + 1].x, x[2 * j + 1].y, x[2 * j + 1].z, x[2 * j + 1].w};
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            c[2 * q] = fmaf(wj, bf16_bits_to_f32(xv[q]), c[2 * q]);
            c[2 * q + 1] = fmaf(wj, bf16_bits_to_f32(xv[q] >> 16), c[2 * q + 1]);
        }
    }
}

// kM4: the block ratio is 4 (two blocks' raw rows are loaded at once); otherwise any ratio.
template <bool kM4, int kVar>
__global__ void __launch_bounds__(kCThreads, 1) pool_index_kernel(
    const uint16_t* __restrict__ raw, const float* __restrict__ gate, const float* __restrict__ bias,
    int m, const float* __restrict__ w_idx, int64_t T, int64_t E, int B, int64_t out_seq_stride,
    uint8_t* __restrict__ kv_out, uint8_t* __restrict__ ikey_out, float* __restrict__ iscale_out, int64_t pos0,
    double rope_base, float inv_scale) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    CompressSmem& sm = *reinterpret_cast<CompressSmem*>(smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023));
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int kWarps = kCThreads / 32;

    if (tid == 0) {
        mbar_init(&sm.mma_done, 1);
        sm.fail = 0;
        fence_barrier_init();
    }
    // per-head keys: four 64-column accumulators (one per head)
    constexpr uint32_t kCols = kVar == kVarPerHead ? 4 * kCTmemCols : kCTmemCols;
    if (warp == 0) {
        tmem_alloc(&sm.tmem_base, kCols);
        tmem_relinquish();
    }
    // W_I^T in bf16, resident for the CTA's lifetime.  It is first needed by the first tile's
    // projection, so it is staged during that tile's pooling: part p (of 4) in pooling iteration
    // p, after the iteration's row loads are issued.  Chunk c (8 per thread) = column n = c % 64
    // and rows k0 = 8 (c / 64) .. k0 + 7 of W_I: 8 loads coalesced across the warp's columns,
    // one 16-byte store of the 8 bf16 values (K-major, 128-byte swizzle).
    // (Per-head keys: each head's W_h^T is staged in turn for every tile, below.)
    constexpr int kWBatch = 32;   // per-head staging: loads per thread in flight at a time
    auto stage_wi_part = [&](int part) {
        if constexpr (kVar == kVarPerHead) return;
        constexpr int kChunks = kDim * kIdxDim / 8 / kCThreads;   // 8 chunks per thread
        constexpr int kPer = kChunks / 4;                          // per pooling iteration
        float v[kPer][8];
#pragma unroll
        for (int q = 0; q < kPer; ++q) {
            const int c = tid + kCThreads * (kPer * part + q);
            const int n = c % kIdxDim, k0 = 8 * (c / kIdxDim);
#pragma unroll
            for (int j = 0; j < 8; ++j) v[q][j] = __ldg(w_idx + (k0 + j) * kIdxDim + n);
        }
#pragma unroll
        for (int q = 0; q < kPer; ++q) {
            const int c = tid + kCThreads * (kPer * part + q);
            const int n = c % kIdxDim, k0 = 8 * (c / kIdxDim);
            *reinterpret_cast<uint4*>(&sm.w[k0 >> 6][sw128(n, 2 * (k0 & 63))]) =
                make_uint4(f32x2_to_bf16x2_bits(v[q][0], v[q][1]), f32x2_to_bf16x2_bits(v[q][2], v[q][3]),
                           f32x2_to_bf16x2_bits(v[q][4], v[q][5]), f32x2_to_bf16x2_bits(v[q][6], v[q][7]));
        }
    };
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    volatile int32_t* fail = &sm.fail;

    // this CTA's entries: an even share [lo, hi) of the B x E entries, walked in tiles of up to
    // kCTile that do not cross a sequence (an even share keeps the longest CTA at ceil(B E /
    // grid) entries instead of two whole tiles when the tile count is not a multiple of the grid)
    const int64_t total = E * B;
    const int64_t lo = total * blockIdx.x / gridDim.x, hi = total * (blockIdx.x + 1) / gridDim.x;
    const float bias_l = (kM4 && lane < 4) ? __ldg(bias + lane) : 0.f;   // slot l's positional bias
    uint32_t phase = 0;
    bool mma_pending = false;   // an MMA reading sm.a was issued and this warp has not seen it end
    bool first_tile = true;
    for (int64_t g0 = lo; g0 < hi;) {
        const int64_t b = g0 / E;
        const int64_t s0 = g0 % E;
        const int n_here = static_cast<int>(min64(min64(kCTile, E - s0), hi - g0));
        g0 += n_here;
        const uint16_t* rb = raw + (size_t)b * T * kDim;
        const float* gb = gate + (size_t)b * T;
        uint8_t* kvb = kv_out + (size_t)b * out_seq_stride * kEntry;

        // ---- 1) pooling: rows warp, warp + 16, ...; kRif rows at a time ------------------
        for (int r0 = warp, it = 0; r0 < kCTile; r0 += kRif * kWarps, ++it) {
            // entries go to the cache as soon as they are pooled; their bf16 copies wait in
            // registers for the shared-memory operand to be free
            uint32_t packed[kRif][8];
            if constexpr (kM4) {
                // the rows and their gates of kRif entries in flight together
                uint4 x[kRif][8];
                float ga[kRif];
#pragma unroll
                for (int h = 0; h < kRif; ++h) {
                    const int r = r0 + h * kWarps;
                    ga[h] = 0.f;
                    if (r < n_here) {
                        load_block4(rb + (size_t)(s0 + r) * 4 * kDim, lane, x[h]);
                        if (lane < 4) ga[h] = __ldg(gb + (s0 + r) * 4 + lane);
                    }
                }
                if (first_tile) stage_wi_part(it);
#pragma unroll
                for (int h = 0; h < kRif; ++h) {
                    const int r = r0 + h * kWarps;
                    float c[16];
                    if (r < n_here) {
                        float w[4];
                        warp_pool_weights_pre(ga[h] + bias_l, 4, lane, w);
                        pool4_preloaded(x[h], w, c);
                        if constexpr (kVar == kVarRope) rope_lane(c, lane, pos0 + (s0 + r + 1) * 4 - 1, rope_base);
                        warp_store_entry<kVar == kVarScaled>(kvb + (size_t)(s0 + r) * kEntry, lane, c, inv_scale);
                    } else {
#pragma unroll
                        for (int d = 0; d < 16; ++d) c[d] = 0.f;
                    }
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        packed[h][q] = f32_to_bf16_bits(c[2 * q]) | (f32_to_bf16_bits(c[2 * q + 1]) << 16);
                }
            } else {
                if (first_tile) stage_wi_part(it);
#pragma unroll 1
                for (int h = 0; h < kRif; ++h) {
                    const int r = r0 + h * kWarps;
                    float c[16];
                    if (r < n_here) {
                        warp_pool<true>(rb + (size_t)(s0 + r) * m * kDim, gb + (s0 + r) * m, bias, m, lane, c);
                        if constexpr (kVar == kVarRope) rope_lane(c, lane, pos0 + (s0 + r + 1) * m - 1, rope_base);
                        warp_store_entry<kVar == kVarScaled>(kvb + (size_t)(s0 + r) * kEntry, lane, c, inv_scale);
                    } else {
#pragma unroll
                        for (int d = 0; d < 16; ++d) c[d] = 0.f;
                    }
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        packed[h][q] = f32_to_bf16_bits(c[2 * q]) | (f32_to_bf16_bits(c[2 * q + 1]) << 16);
                }
            }
            // the previous tile's MMA must be done reading sm.a before the first write
            if (mma_pending) {
                if (!mbar_wait(&sm.mma_done, phase ^ 1u)) *fail = 1;
                mma_pending = false;
            }
#pragma unroll
            for (int h = 0; h < kRif; ++h) {
                const int r = r0 + h * kWarps;
                // lane l holds dims 16l..16l+15: column block l / 4, bytes 32 (l % 4) .. +31
                uint8_t* blk = sm.a[lane >> 2];
                const int cb = 32 * (lane & 3);
                *reinterpret_cast<uint4*>(blk + sw128(r, cb)) =
                    make_uint4(packed[h][0], packed[h][1], packed[h][2], packed[h][3]);
                *reinterpret_cast<uint4*>(blk + sw128(r, cb + 16)) =
                    make_uint4(packed[h][4], packed[h][5], packed[h][6], packed[h][7]);
            }
        }
        first_tile = false;
        fence_proxy_async_smem();   // the pooled rows (and, after the first tile, W_I) for the MMA
        tc_fence_before();
        __syncthreads();
        if (*fail) break;
        if constexpr (kVar == kVarPerHead) {
            // ---- 2') per head h: W_h^T staged (the previous head's MMA has ended), one MMA chain
            //      into columns 64h..64h+63 --------------------------------------------------------
            bool ok = true;
            for (int h = 0; h < kIdxHeads && ok; ++h) {
                for (int i0 = 0; i0 < kDim * kIdxDim; i0 += kWBatch * kCThreads) {
                    float v[kWBatch];
#pragma unroll
                    for (int u = 0; u < kWBatch; ++u) {
                        const int i = i0 + u * kCThreads + tid;
                        v[u] = __ldg(w_idx + (size_t)(i / kIdxDim) * kIdxHeads * kIdxDim + h * kIdxDim + i % kIdxDim);
                    }
#pragma unroll
                    for (int u = 0; u < kWBatch; ++u) {
                        const int i = i0 + u * kCThreads + tid;
                        const int k = i / kIdxDim, n = i % kIdxDim;
                        *reinterpret_cast<uint16_t*>(&sm.w[k >> 6][sw128(n, 2 * (k & 63))]) =
                            static_cast<uint16_t>(f32_to_bf16_bits(v[u]));
                    }
                }
                fence_proxy_async_smem();
                tc_fence_before();
                __syncthreads();
                if (tid == 0) {
                    tc_fence_after();
#pragma unroll
                    for (int kb = 0; kb < kDim / 64; ++kb)
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks)
                            umma_f16(tmem + static_cast<uint32_t>(kIdxDim * h), desc_sw128(sm.a[kb], 0) + (32 * ks) / 16,
                                     desc_sw128(sm.w[kb], 0) + (32 * ks) / 16, kIdProj, (kb | ks) != 0 ? 1u : 0u);
                    umma_commit(&sm.mma_done);
                }
                ok = !__syncthreads_or(!mbar_wait(&sm.mma_done, phase));
                phase ^= 1u;
                tc_fence_after();
            }
            if (!ok) {
                if (tid == 0) *fail = 1;
                break;
            }
            // ---- 3') FP4 keys of the four heads: warps 0-3, thread = entry -------------------
            if (warp < 4) {
                // every lane reads tensor memory (the loads are warp-wide); only the tile's
                // entries are stored
                const int r = 32 * warp + lane;
                const int64_t s = s0 + r;
                const bool store = r < n_here;
                uint8_t* kdst = ikey_out + ((size_t)b * out_seq_stride + (size_t)s) * kIkeyHead;
                float* sdst = iscale_out + ((size_t)b * out_seq_stride + (size_t)s) * (2 * kIdxHeads);
                const int sw = static_cast<int>(s & 7);
#pragma unroll 1
                for (int h = 0; h < kIdxHeads; ++h) {
#pragma unroll
                    for (int g = 0; g < 2; ++g) {
                        uint32_t u[2][16];
                        const uint32_t col = static_cast<uint32_t>(kIdxDim * h + 32 * g);
                        tmem_ld_32x32b_x16(tmem + ((32u * warp) << 16) + col, u[0]);
                        tmem_ld_32x32b_x16(tmem + ((32u * warp) << 16) + col + 16u, u[1]);
                        tmem_ld_wait();
                        float sc;
                        uint32_t words[4];
                        fp4_group_words(u, &sc, words);
                        // chunk 2h + g of the entry's 128-byte row, at chunk (2h + g) ^ (s mod 8)
                        if (store) {
                            *reinterpret_cast<uint4*>(kdst + 16 * ((2 * h + g) ^ sw)) =
                                make_uint4(words[0], words[1], words[2], words[3]);
                            sdst[2 * h + g] = sc;
                        }
                    }
                }
                tc_fence_before();
            }
            continue;
        }
        // ---- 2) projection on the tensor cores ---------------------------------------------
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kb = 0; kb < kDim / 64; ++kb)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)   // 16 bf16 = 32 bytes of K per MMA
                    umma_f16(tmem, desc_sw128(sm.a[kb], 0) + (32 * ks) / 16, desc_sw128(sm.w[kb], 0) + (32 * ks) / 16,
                             kIdProj, (kb | ks) != 0 ? 1u : 0u);
            umma_commit(&sm.mma_done);
        }
        mma_pending = true;
        // ---- 3) FP4 keys: warps 0-7, thread = entry; warps 0-3 quantise group 0 (columns
        //      0..31), warps 4-7 group 1 (columns 32..63) of their lane quarter's entries -------
        if (warp < 8) {
            const bool ok = mbar_wait(&sm.mma_done, phase);
            mma_pending = false;
            if (!ok) *fail = 1;
            tc_fence_after();
            const int quarter = warp & 3, g = warp >> 2;
            const int r = 32 * quarter + lane;
            const int64_t s = s0 + r;
            const int sw = static_cast<int>((s >> 2) & 1);
            const bool store = ok && r < n_here;
            uint32_t u[2][16];
            tmem_ld_32x32b_x16(tmem + ((32u * quarter) << 16) + 32u * g, u[0]);
            tmem_ld_32x32b_x16(tmem + ((32u * quarter) << 16) + 32u * g + 16u, u[1]);
            tmem_ld_wait();
            tc_fence_before();
            float amax = 0.f;
#pragma unroll
            for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(__uint_as_float(u[i >> 4][i & 15])));
            const float sc = fp4_group_scale(amax);
            const float inv = 1.0f / sc;   // exact: a power of two
            uint32_t words[4];
#pragma unroll
            for (int wq = 0; wq < 4; ++wq) {
                uint32_t word = 0u;
#pragma unroll
                for (int bq = 0; bq < 4; ++bq) {
                    const int i = 8 * wq + 2 * bq;   // elements i, i+1 of the group
                    const uint32_t byte = e2m1_code(__uint_as_float(u[i >> 4][i & 15]) * inv) |
                                          (e2m1_code(__uint_as_float(u[(i + 1) >> 4][(i + 1) & 15]) * inv) << 4);
                    word |= byte << (8 * bq);
                }
                words[wq] = word;
            }
            // group g's 16 bytes go to half g XOR (bit 2 of s) of the stored key
            if (store) {
                reinterpret_cast<uint4*>(ikey_out + ((size_t)b * out_seq_stride + (size_t)s) * kIkey)[g ^ sw] =
                    make_uint4(words[0], words[1], words[2], words[3]);
                iscale_out[((size_t)b * out_seq_stride + (size_t)s) * 2 + g] = sc;
            }
        }
        phase ^= 1u;
    }
    // the last MMA (if any) must end before tensor memory is released
    if (mma_pending && tid == 0) (void)mbar_wait(&sm.mma_done, phase ^ 1u);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kCols);
    }
}

size_t compress_index_smem_bytes() { return sizeof(CompressSmem) + 1024; }

cudaError_t launch_compress(const uint16_t* raw, const float* gate, const float* bias, int m,
                            const float* w_idx, int64_t T, int B, int64_t out_seq_stride,
                            uint8_t* kv_out, uint8_t* ikey_out, float* iscale_out, int num_sms,
                            cudaStream_t stream, int64_t pos0, double rope_base, float kv_scale, bool perhead) {
    const int64_t E = T / m;
    if (E <= 0 || B <= 0) return cudaSuccess;
    const int var = perhead ? kVarPerHead : (rope_base > 0.0 ? kVarRope : (kv_scale != 1.f ? kVarScaled : kVarBase));
    const float inv_scale = 1.f / kv_scale;
    if (w_idx == nullptr) {
        const int64_t warps = E * B;
        const int64_t blocks = (warps + 7) / 8;
        auto kernel = var == kVarRope ? pool_kernel<kVarRope> : (var == kVarScaled ? pool_kernel<kVarScaled> : pool_kernel<kVarBase>);
        kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(raw, gate, bias, m, T, E, B, out_seq_stride, kv_out,
                                                                  pos0, rope_base, inv_scale);
        return cudaGetLastError();
    }
    const size_t smem = compress_index_smem_bytes();
    const int64_t tiles = ((E + kCTile - 1) / kCTile) * B;
    const int64_t grid = min64(tiles, num_sms);
    auto kernel = (m == 4) ? (var == kVarRope ? pool_index_kernel<true, kVarRope>
                                              : (var == kVarScaled ? pool_index_kernel<true, kVarScaled>
                                                 : (var == kVarPerHead ? pool_index_kernel<true, kVarPerHead>
                                                                       : pool_index_kernel<true, kVarBase>)))
                           : (var == kVarRope ? pool_index_kernel<false, kVarRope>
                                              : (var == kVarScaled ? pool_index_kernel<false, kVarScaled>
                                                 : (var == kVarPerHead ? pool_index_kernel<false, kVarPerHead>
                                                                       : pool_index_kernel<false, kVarBase>)));
    cudaError_t e = set_smem_once(kernel, smem);
    if (e != cudaSuccess) return e;
    kernel<<<static_cast<unsigned>(grid), kCThreads, smem, stream>>>(raw, gate, bias, m, w_idx, T, E, B, out_seq_stride,
                                                                     kv_out, ikey_out, iscale_out, pos0, rope_base,
                                                                     inv_scale);
    return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------
// Per-channel gating (a layout / gating variant): one gate logit per token and dimension and one
// bias per block slot and dimension; every dimension d of entry s pools its own softmax,
//   a_j = gate[s m + j][d] + bias[j][d],  w = softmax_j(a),  c_d = sum_j w_j x[s m + j][d].
// One warp per entry (lane l: dims 16l..16l+15), an online softmax over the slots in order, four
// slots' loads in flight.  With w_idx the indexer key is projected on the CUDA cores from bf16
// operands (W_I^T staged in shared memory) and FP4-quantised as for csld_compress.
// ------------------------------------------------------------------------------------------
constexpr int kChThreads = 256;
struct ChannelSmem {
    uint16_t wt[kIdxDim][kDim];       // W_I^T, bf16
    float c[kChThreads / 32][kDim];   // each warp's pooled entry
};

__global__ void __launch_bounds__(kChThreads) pool_channel_kernel(
    const uint16_t* __restrict__ raw, const float* __restrict__ gate, const float* __restrict__ bias, int m,
    const float* __restrict__ w_idx, int64_t T, int64_t E, uint8_t* __restrict__ kv_out, uint8_t* __restrict__ ikey_out,
    float* __restrict__ iscale_out) {
    extern __shared__ __align__(16) uint8_t ch_raw[];
    ChannelSmem& sm = *reinterpret_cast<ChannelSmem*>(ch_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (w_idx) {
        for (int i = tid; i < kDim * kIdxDim; i += kChThreads) {
            const int k = i / kIdxDim, n = i % kIdxDim;
            sm.wt[n][k] = static_cast<uint16_t>(f32_to_bf16_bits(__ldg(w_idx + i)));
        }
        __syncthreads();
    }
    const int64_t n_warps = (int64_t)gridDim.x * (kChThreads / 32);
    for (int64_t s = (int64_t)blockIdx.x * (kChThreads / 32) + warp; s < E; s += n_warps) {
        float mx[16], sum[16], acc[16];
#pragma unroll
        for (int d = 0; d < 16; ++d) {
            mx[d] = -INFINITY;
            sum[d] = 0.f;
            acc[d] = 0.f;
        }
        const size_t t0 = (size_t)s * m;
        for (int j0 = 0; j0 < m; j0 += 4) {
            uint4 x[4][2];
            float4 g[4][4], bb[4][4];
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                if (j0 + r < m) {
                    const size_t t = t0 + j0 + r;
                    const uint4* xr = reinterpret_cast<const uint4*>(raw + t * kDim) + 2 * lane;
                    const float4* gr = reinterpret_cast<const float4*>(gate + t * kDim) + 4 * lane;
                    const float4* br = reinterpret_cast<const float4*>(bias + (size_t)(j0 + r) * kDim) + 4 * lane;
                    x[r][0] = __ldg(xr);
                    x[r][1] = __ldg(xr + 1);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        g[r][q] = __ldg(gr + q);
                        bb[r][q] = __ldg(br + q);
                    }
                }
            }
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                if (j0 + r >= m) break;
                const uint32_t xv[8] = {x[r][0].x, x[r][0].y, x[r][0].z, x[r][0].w,
                                        x[r][1].x, x[r][1].y, x[r][1].z, x[r][1].w};
                const float gv[16] = {g[r][0].x, g[r][0].y, g[r][0].z, g[r][0].w, g[r][1].x, g[r][1].y, g[r][1].z,
                                      g[r][1].w, g[r][2].x, g[r][2].y, g[r][2].z, g[r][2].w, g[r][3].x, g[r][3].y,
                                      g[r][3].z, g[r][3].w};
                const float bv[16] = {bb[r][0].x, bb[r][0].y, bb[r][0].z, bb[r][0].w, bb[r][1].x, bb[r][1].y,
                                      bb[r][1].z, bb[r][1].w, bb[r][2].x, bb[r][2].y, bb[r][2].z, bb[r][2].w,
                                      bb[r][3].x, bb[r][3].y, bb[r][3].z, bb[r][3].w};
#pragma unroll
                for (int d = 0; d < 16; ++d) {
                    const float a = gv[d] + bv[d];
                    const float xd = bf16_bits_to_f32(d & 1 ? xv[d >> 1] >> 16 : xv[d >> 1]);
                    if (a > mx[d]) {   // a new maximum: rescale what was accumulated
                        const float f = expf(mx[d] - a);
                        sum[d] = fmaf(sum[d], f, 1.f);
                        acc[d] = fmaf(acc[d], f, xd);
                        mx[d] = a;
                    } else {
                        const float e = expf(a - mx[d]);
                        sum[d] += e;
                        acc[d] = fmaf(e, xd, acc[d]);
                    }
                }
            }
        }
        float c[16];
#pragma unroll
        for (int d = 0; d < 16; ++d) c[d] = acc[d] / sum[d];
        warp_store_entry(kv_out + (size_t)s * kEntry, lane, c);
        if (w_idx) {
            // u_j = sum_d bf16(c_d) * bf16(W_I[d][j]) in fp32; lane l forms u_{2l}, u_{2l+1}
#pragma unroll
            for (int d = 0; d < 16; ++d) sm.c[warp][16 * lane + d] = bf16_bits_to_f32(f32_to_bf16_bits(c[d]));
            __syncwarp();
            float u0 = 0.f, u1 = 0.f;
            for (int d = 0; d < kDim; ++d) {
                const float cd = sm.c[warp][d];
                u0 = fmaf(cd, bf16_bits_to_f32(sm.wt[2 * lane][d]), u0);
                u1 = fmaf(cd, bf16_bits_to_f32(sm.wt[2 * lane + 1][d]), u1);
            }
            __syncwarp();
            warp_store_fp4(ikey_out + (size_t)s * kIkey, iscale_out + (size_t)s * 2, s, lane, u0, u1);
        }
    }
}

cudaError_t launch_compress_channel(const uint16_t* raw, const float* gate, const float* bias, int m,
                                    const float* w_idx, int64_t T, uint8_t* kv_out, uint8_t* ikey_out,
                                    float* iscale_out, int num_sms, cudaStream_t stream) {
    const int64_t E = T / m;
    if (E <= 0) return cudaSuccess;
    const size_t smem = w_idx ? sizeof(ChannelSmem) : 0;
    cudaError_t e = set_smem_once(pool_channel_kernel, sizeof(ChannelSmem));
    if (e != cudaSuccess) return e;
    const int64_t blocks = min64((E + kChThreads / 32 - 1) / (kChThreads / 32), 4LL * num_sms);
    pool_channel_kernel<<<static_cast<unsigned>(blocks), kChThreads, smem, stream>>>(raw, gate, bias, m, w_idx, T, E,
                                                                                    kv_out, ikey_out, iscale_out);
    return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------
// Window ring + tail after a prefill of T tokens (one CTA per sequence).
// ------------------------------------------------------------------------------------------
template <int kVar>
__global__ void __launch_bounds__(128) prefill_state_kernel(const uint16_t* __restrict__ raw,
                                                            const float* __restrict__ gate,
                                                            int64_t T, int m, int W,
                                                            uint8_t* __restrict__ win_kv,
                                                            uint16_t* __restrict__ tail_kv,
                                                            float* __restrict__ tail_gate,
                                                            int32_t* __restrict__ seq_len, double rope_base,
                                                            float inv_scale) {
    const int b = blockIdx.x, tid = threadIdx.x;
    const uint16_t* rb = raw + (size_t)b * T * kDim;
    // window: tokens max(0, T-W) .. T-1; thread handles 4 dims (8 bytes of bf16)
    const int64_t w0 = max64(0, T - W);
    for (int64_t t = w0; t < T; ++t) {
        const uint2 x = *reinterpret_cast<const uint2*>(rb + (size_t)t * kDim + 4 * tid);
        uint8_t* e = win_kv + ((size_t)b * W + (size_t)(t % W)) * kEntry;
        if (tid < kNope / 4) {
            *reinterpret_cast<uint32_t*>(e + 4 * tid) = fp8x4_of_bf16x4<kVar == kVarScaled>(x, inv_scale);
        } else {
            uint2 y = x;
            if constexpr (kVar == kVarRope) y = rope_bf16x4(x, tid - kNope / 4, t, rope_base);   // at token t
            *reinterpret_cast<uint2*>(e + kNope + 8 * (tid - kNope / 4)) = y;
        }
    }
    const int64_t t0 = T - (T % m);
    for (int64_t t = t0; t < T; ++t) {
        *reinterpret_cast<uint2*>(tail_kv + ((size_t)b * m + (size_t)(t % m)) * kDim + 4 * tid) =
            *reinterpret_cast<const uint2*>(rb + (size_t)t * kDim + 4 * tid);
        if (tid == 0) tail_gate[(size_t)b * m + (size_t)(t % m)] = gate[(size_t)b * T + t];
    }
    if (tid == 0) seq_len[b] = static_cast<int32_t>(T);
}

cudaError_t launch_prefill_state(const uint16_t* raw, const float* gate, int64_t T, int m, int W,
                                 int B, uint8_t* win_kv, uint16_t* tail_kv, float* tail_gate,
                                 int32_t* seq_len, cudaStream_t stream, double rope_base, float kv_scale) {
    auto kernel = rope_base > 0.0 ? prefill_state_kernel<kVarRope>
                                  : (kv_scale != 1.f ? prefill_state_kernel<kVarScaled> : prefill_state_kernel<kVarBase>);
    kernel<<<B, 128, 0, stream>>>(raw, gate, T, m, W, win_kv, tail_kv, tail_gate, seq_len, rope_base, 1.f / kv_scale);
    return cudaGetLastError();
}

}  // namespace csld

namespace csld {

// ------------------------------------------------------------------------------------------
// Decode-time append of one token per sequence (one CTA of 256 threads per sequence).
// Token t = seq_len[b] goes to window slot t mod W and tail slot t mod m; when it completes a
// block, the m tail rows are pooled with the same warp routine as the prefill (so the entry
// bytes match csld_compress bit for bit) and, for CSA, projected and FP4-quantised.
// ------------------------------------------------------------------------------------------
constexpr int kAppendThreads = 256;

template <int kVar>
__global__ void __launch_bounds__(kAppendThreads) append_kernel(csld_layer_cache cache,
                                                                const uint16_t* __restrict__ kv_new,
                                                                const float* __restrict__ gate_new,
                                                                int32_t* err, double rope_base, float inv_scale) {
    __shared__ float cbuf[kDim];
    __shared__ float upart[kAppendThreads / 32][kIdxDim];
    const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    pdl_wait();      // the token and the cache come from upstream
    pdl_trigger();
    const int m = cache.ratio, W = cache.window;
    const int64_t cap = cache.capacity;
    const int32_t t = cache.seq_len[b];
    if (t < 0) {
        if (tid == 0) dev_error(err, CSLD_DEVERR_SEQ_LEN);
        return;
    }
    const bool complete = ((t + 1) % m) == 0;
    const int64_t s = t / m;
    if (complete && s >= cap) {
        if (tid == 0) dev_error(err, CSLD_DEVERR_CAPACITY);
        return;
    }
    // threads 0..127 move the token (4 dims each); all 256 share the block's projection
    const bool mover = tid < kDim / 4;
    const uint2 x = mover ? *reinterpret_cast<const uint2*>(kv_new + (size_t)b * kDim + 4 * tid) : make_uint2(0u, 0u);
    if (W > 0 && mover) {
        uint8_t* e = cache.win_kv + ((size_t)b * W + (size_t)(t % W)) * kEntry;
        if (tid < kNope / 4) {
            *reinterpret_cast<uint32_t*>(e + 4 * tid) = fp8x4_of_bf16x4<kVar == kVarScaled>(x, inv_scale);
        } else {
            uint2 y = x;
            if constexpr (kVar == kVarRope) y = rope_bf16x4(x, tid - kNope / 4, t, rope_base);   // at token t
            *reinterpret_cast<uint2*>(e + kNope + 8 * (tid - kNope / 4)) = y;
        }
    }
    uint16_t* tail = cache.tail_kv + (size_t)b * m * kDim;
    float* tgate = cache.tail_gate + (size_t)b * m;
    if (mover) *reinterpret_cast<uint2*>(tail + (size_t)(t % m) * kDim + 4 * tid) = x;
    if (tid == 0) tgate[t % m] = gate_new[b];
    if (complete) {
        __syncthreads();  // the new tail row and gate are visible to the whole block
        if (warp == 0) {
            float c[16];
            warp_pool<false>(tail, tgate, cache.pos_bias, m, lane, c);
            if constexpr (kVar == kVarRope) rope_lane(c, lane, t, rope_base);   // token t ends the block
            warp_store_entry<kVar == kVarScaled>(cache.comp_kv + ((size_t)b * cap + (size_t)s) * kEntry, lane, c,
                                                 inv_scale);
#pragma unroll
            for (int d = 0; d < 16; ++d) cbuf[16 * lane + d] = bf16_bits_to_f32(f32_to_bf16_bits(c[d]));
        }
        if (kVar == kVarPerHead && cache.has_indexer) {
            // per-head keys: the same projection for each head h with W_h (W_I [512][4][64])
            __syncthreads();
#pragma unroll 1
            for (int h = 0; h < kIdxHeads; ++h) {
                float a0 = 0.f, a1 = 0.f;
                const float* wrow = cache.w_idx + (size_t)(64 * warp) * kIdxHeads * kIdxDim + h * kIdxDim;
#pragma unroll 16
                for (int d = 0; d < 64; ++d) {
                    const float cd = cbuf[64 * warp + d];
                    const float* wr = wrow + (size_t)d * kIdxHeads * kIdxDim;
                    a0 = fmaf(cd, bf16_bits_to_f32(f32_to_bf16_bits(__ldg(wr + lane))), a0);
                    a1 = fmaf(cd, bf16_bits_to_f32(f32_to_bf16_bits(__ldg(wr + 32 + lane))), a1);
                }
                upart[warp][lane] = a0;
                upart[warp][32 + lane] = a1;
                __syncthreads();
                if (warp == 0) {
                    float u0 = 0.f, u1 = 0.f;
#pragma unroll
                    for (int w = 0; w < kAppendThreads / 32; ++w) {
                        u0 += upart[w][2 * lane];
                        u1 += upart[w][2 * lane + 1];
                    }
                    warp_store_fp4_head(cache.ikeys + ((size_t)b * cap + (size_t)s) * kIkeyHead,
                                        cache.iscales + ((size_t)b * cap + (size_t)s) * (2 * kIdxHeads), s, h, lane, u0,
                                        u1);
                }
                __syncthreads();   // upart is written again for the next head
            }
        } else if (cache.has_indexer) {
            __syncthreads();
            // u_j = sum_d bf16(c_d) * bf16(W_I[d][j]) in fp32 (the operands the prefill
            // projection feeds its tensor cores).  Warp w takes dims 64w..64w+63, lane outputs
            // lane and lane + 32: every W_I load is independent and warp-coalesced.
            float a0 = 0.f, a1 = 0.f;
            const float* wrow = cache.w_idx + (size_t)(64 * warp) * kIdxDim;
#pragma unroll 16
            for (int d = 0; d < 64; ++d) {
                const float cd = cbuf[64 * warp + d];
                a0 = fmaf(cd, bf16_bits_to_f32(f32_to_bf16_bits(__ldg(wrow + (size_t)d * kIdxDim + lane))), a0);
                a1 = fmaf(cd, bf16_bits_to_f32(f32_to_bf16_bits(__ldg(wrow + (size_t)d * kIdxDim + 32 + lane))), a1);
            }
            upart[warp][lane] = a0;
            upart[warp][32 + lane] = a1;
            __syncthreads();
            if (warp == 0) {
                float u0 = 0.f, u1 = 0.f;
#pragma unroll
                for (int w = 0; w < kAppendThreads / 32; ++w) {
                    u0 += upart[w][2 * lane];
                    u1 += upart[w][2 * lane + 1];
                }
                warp_store_fp4(cache.ikeys + ((size_t)b * cap + (size_t)s) * kIkey,
                               cache.iscales + ((size_t)b * cap + (size_t)s) * 2, s, lane, u0, u1);
            }
        }
    }
    if (tid == 0) cache.seq_len[b] = t + 1;
}

cudaError_t launch_append(const csld_layer_cache& cache, const uint16_t* kv_new,
                          const float* gate_new, int32_t* err, cudaStream_t stream, double rope_base,
                          float kv_scale, bool perhead) {
    auto kernel = perhead ? append_kernel<kVarPerHead>
                          : (rope_base > 0.0 ? append_kernel<kVarRope>
                                             : (kv_scale != 1.f ? append_kernel<kVarScaled> : append_kernel<kVarBase>));
    cudaError_t e = launch_pdl(kernel, dim3(cache.batch), dim3(kAppendThreads), 0, stream, cache, kv_new, gate_new, err,
                               rope_base, 1.f / kv_scale);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace csld
