// Prefill compression: softmax-gated pooling with a learned positional bias into 576-byte
// FP8/bf16 entries, plus the FP4 lightning-indexer key of each CSA entry.
//
// Source: "DeepSeek-V4: a million-token context that agents can actually use" -- CSA paragraph
// and Figure 3 caption (4 tokens -> one entry by softmax-gated pooling with a positional bias;
// FP4 lightning indexer over the compressed entries), HCA paragraph and Figure 4 caption (128
// tokens -> one entry), storage paragraph (FP8 entries, bf16 RoPE dims, FP4 indexer).
//
// Layout: one warp pools one entry; lane l owns dims [16l, 16l+16).  The raw stream is read
// once with 16-byte loads (HBM-bound).  For CSA the pooled vectors of a 32-entry tile are
// staged as bf16 in shared memory and projected by W_I (512x64, bf16 copy resident in shared
// memory for the whole persistent CTA) on the tensor cores (mma.sync m16n8k16, fp32
// accumulation); the FP4 quantisation runs on the fp32 result.
#include "csld_internal.cuh"
#include "kernels.cuh"

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
template <bool kReadOnly>
__device__ __forceinline__ void warp_pool(const uint16_t* rows, const float* gate,
                                          const float* __restrict__ bias, int m, int lane,
                                          float (&c)[16]) {
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
    float w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] = e[i] / s;

#pragma unroll
    for (int d = 0; d < 16; ++d) c[d] = 0.f;
    const uint4* base = reinterpret_cast<const uint4*>(rows) + 2 * lane;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if (32 * i >= m) break;
        const int jn = min(32, m - 32 * i);
        int jj = 0;
        // two rows per iteration keep four 16-byte loads in flight per lane
        for (; jj + 1 < jn; jj += 2) {
            const int j = 32 * i + jj;
            const uint4 x0 = load_row16<kReadOnly>(base + (size_t)j * (kDim / 8));
            const uint4 x1 = load_row16<kReadOnly>(base + (size_t)j * (kDim / 8) + 1);
            const uint4 y0 = load_row16<kReadOnly>(base + (size_t)(j + 1) * (kDim / 8));
            const uint4 y1 = load_row16<kReadOnly>(base + (size_t)(j + 1) * (kDim / 8) + 1);
            const float wj = __shfl_sync(0xffffffffu, w[i], jj);
            const float wk = __shfl_sync(0xffffffffu, w[i], jj + 1);
            const uint32_t xv[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
            const uint32_t yv[8] = {y0.x, y0.y, y0.z, y0.w, y1.x, y1.y, y1.z, y1.w};
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                c[2 * q] = fmaf(wj, bf16_bits_to_f32(xv[q]), c[2 * q]);
                c[2 * q + 1] = fmaf(wj, bf16_bits_to_f32(xv[q] >> 16), c[2 * q + 1]);
            }
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                c[2 * q] = fmaf(wk, bf16_bits_to_f32(yv[q]), c[2 * q]);
                c[2 * q + 1] = fmaf(wk, bf16_bits_to_f32(yv[q] >> 16), c[2 * q + 1]);
            }
        }
        for (; jj < jn; ++jj) {
            const int j = 32 * i + jj;
            const uint4 x0 = load_row16<kReadOnly>(base + (size_t)j * (kDim / 8));
            const uint4 x1 = load_row16<kReadOnly>(base + (size_t)j * (kDim / 8) + 1);
            const float wj = __shfl_sync(0xffffffffu, w[i], jj);
            const uint32_t xv[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                c[2 * q] = fmaf(wj, bf16_bits_to_f32(xv[q]), c[2 * q]);
                c[2 * q + 1] = fmaf(wj, bf16_bits_to_f32(xv[q] >> 16), c[2 * q + 1]);
            }
        }
    }
}

// Writes the 576-byte entry of the pooled vector held by the warp (lane l: dims 16l..16l+15).
__device__ __forceinline__ void warp_store_entry(uint8_t* __restrict__ entry, int lane,
                                                 const float (&c)[16]) {
    if (lane < kNope / 16) {
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
            w[q] = f32_to_e4m3(c[4 * q]) | (f32_to_e4m3(c[4 * q + 1]) << 8) |
                   (f32_to_e4m3(c[4 * q + 2]) << 16) | (f32_to_e4m3(c[4 * q + 3]) << 24);
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

// ------------------------------------------------------------------------------------------
// Pooling without an indexer key (HCA, or any ratio).  One warp per entry.
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) pool_kernel(const uint16_t* __restrict__ raw,
                                                   const float* __restrict__ gate,
                                                   const float* __restrict__ bias, int m,
                                                   int64_t T, int64_t E, int B,
                                                   int64_t out_seq_stride,
                                                   uint8_t* __restrict__ kv_out) {
    const int lane = threadIdx.x & 31;
    const int64_t gw = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (gw >= E * B) return;
    const int64_t b = gw / E, s = gw % E;
    float c[16];
    warp_pool<true>(raw + ((size_t)b * T + (size_t)s * m) * kDim, gate + (size_t)b * T + (size_t)s * m,
              bias, m, lane, c);
    warp_store_entry(kv_out + ((size_t)b * out_seq_stride + (size_t)s) * kEntry, lane, c);
}

// ------------------------------------------------------------------------------------------
// Pooling + indexer key (CSA).  Persistent CTAs of 8 warps over 32-entry tiles.
// ------------------------------------------------------------------------------------------
constexpr int kCTile = 32;                 // entries per tile
constexpr int kAStride = kDim + 8;         // bf16 elements per staged row (16-byte pad)
constexpr int kWStride = kDim + 8;         // bf16 elements per W^T row
constexpr int kUStride = kIdxDim + 4;      // floats per projected row

struct CompressSmem {
    uint16_t wt[kIdxDim * kWStride];       // W_I^T in bf16: wt[n][k] = bf16(W_I[k][n])
    uint16_t a[kCTile * kAStride];         // pooled rows of the tile, bf16
    float u[kCTile * kUStride];            // projected rows, fp32
};

__global__ void __launch_bounds__(256) pool_index_kernel(
    const uint16_t* __restrict__ raw, const float* __restrict__ gate, const float* __restrict__ bias,
    int m, const float* __restrict__ w_idx, int64_t T, int64_t E, int B, int64_t out_seq_stride,
    uint8_t* __restrict__ kv_out, uint8_t* __restrict__ ikey_out, float* __restrict__ iscale_out) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    CompressSmem& sm = *reinterpret_cast<CompressSmem*>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    // W_I^T (bf16) resident for the CTA's lifetime.
    for (int i = tid; i < kDim * kIdxDim; i += blockDim.x) {
        const int k = i / kIdxDim, n = i % kIdxDim;
        sm.wt[n * kWStride + k] = static_cast<uint16_t>(f32_to_bf16_bits(w_idx[i]));
    }

    const int64_t tiles_per_seq = (E + kCTile - 1) / kCTile;
    const int64_t n_tiles = tiles_per_seq * B;
    for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
        const int64_t b = tile / tiles_per_seq;
        const int64_t s0 = (tile % tiles_per_seq) * kCTile;
        const int n_here = static_cast<int>(min64(kCTile, E - s0));
        __syncthreads();  // previous tile's smem fully consumed (and W^T written on the first pass)

        // 1) pool 4 entries per warp; store entries; stage bf16 rows
        for (int r = warp; r < kCTile; r += 8) {
            uint32_t packed[8];
            if (r < n_here) {
                const int64_t s = s0 + r;
                float c[16];
                warp_pool<true>(raw + ((size_t)b * T + (size_t)s * m) * kDim,
                          gate + (size_t)b * T + (size_t)s * m, bias, m, lane, c);
                warp_store_entry(kv_out + ((size_t)b * out_seq_stride + (size_t)s) * kEntry, lane, c);
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    packed[q] = f32_to_bf16_bits(c[2 * q]) | (f32_to_bf16_bits(c[2 * q + 1]) << 16);
            } else {
#pragma unroll
                for (int q = 0; q < 8; ++q) packed[q] = 0u;
            }
            uint4* dst = reinterpret_cast<uint4*>(&sm.a[r * kAStride + 16 * lane]);
            dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
            dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
        }
        __syncthreads();

        // 2) u[32][64] = A[32][512] . W[512][64]; warp w: m-tile (w&1), n-tiles 2*(w>>1)+{0,1}
        {
            const int mt = warp & 1, nt0 = 2 * (warp >> 1);
            const int g = lane >> 2, cq = lane & 3;
            float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
            // ldmatrix addresses: lanes 0-15 rows 0-15 (k 0..7), lanes 16-31 rows 0-15 (k 8..15)
            const uint16_t* arow = &sm.a[(mt * 16 + (lane & 15)) * kAStride + ((lane >> 4) << 3)];
#pragma unroll 4
            for (int ks = 0; ks < kDim / 16; ++ks) {
                uint32_t a0, a1, a2, a3;
                ldmatrix_x4(a0, a1, a2, a3, arow + ks * 16);
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const uint16_t* wr = &sm.wt[((nt0 + j) * 8 + g) * kWStride + ks * 16 + 2 * cq];
                    const uint32_t b0 = *reinterpret_cast<const uint32_t*>(wr);
                    const uint32_t b1 = *reinterpret_cast<const uint32_t*>(wr + 8);
                    mma_bf16(acc[j], a0, a1, a2, a3, b0, b1);
                }
            }
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int col = (nt0 + j) * 8 + 2 * cq;
                sm.u[(mt * 16 + g) * kUStride + col] = acc[j][0];
                sm.u[(mt * 16 + g) * kUStride + col + 1] = acc[j][1];
                sm.u[(mt * 16 + g + 8) * kUStride + col] = acc[j][2];
                sm.u[(mt * 16 + g + 8) * kUStride + col + 1] = acc[j][3];
            }
        }
        __syncthreads();

        // 3) FP4 keys
        for (int r = warp; r < n_here; r += 8) {
            const int64_t s = s0 + r;
            const float u0 = sm.u[r * kUStride + 2 * lane];
            const float u1 = sm.u[r * kUStride + 2 * lane + 1];
            warp_store_fp4(ikey_out + ((size_t)b * out_seq_stride + (size_t)s) * kIkey,
                           iscale_out + ((size_t)b * out_seq_stride + (size_t)s) * 2, s, lane, u0, u1);
        }
    }
}

size_t compress_index_smem_bytes() { return sizeof(CompressSmem); }

cudaError_t launch_compress(const uint16_t* raw, const float* gate, const float* bias, int m,
                            const float* w_idx, int64_t T, int B, int64_t out_seq_stride,
                            uint8_t* kv_out, uint8_t* ikey_out, float* iscale_out, int num_sms,
                            cudaStream_t stream) {
    const int64_t E = T / m;
    if (E <= 0 || B <= 0) return cudaSuccess;
    if (w_idx == nullptr) {
        const int64_t warps = E * B;
        const int64_t blocks = (warps + 7) / 8;
        pool_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(raw, gate, bias, m, T, E, B,
                                                                       out_seq_stride, kv_out);
        return cudaGetLastError();
    }
    const size_t smem = sizeof(CompressSmem);
    cudaError_t e = set_smem_once(pool_index_kernel, smem);
    if (e != cudaSuccess) return e;
    const int64_t tiles = ((E + kCTile - 1) / kCTile) * B;
    const int64_t grid = min64(tiles, 2LL * num_sms);
    pool_index_kernel<<<static_cast<unsigned>(grid), 256, smem, stream>>>(
        raw, gate, bias, m, w_idx, T, E, B, out_seq_stride, kv_out, ikey_out, iscale_out);
    return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------
// Window ring + tail after a prefill of T tokens (one CTA per sequence).
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(128) prefill_state_kernel(const uint16_t* __restrict__ raw,
                                                            const float* __restrict__ gate,
                                                            int64_t T, int m, int W,
                                                            uint8_t* __restrict__ win_kv,
                                                            uint16_t* __restrict__ tail_kv,
                                                            float* __restrict__ tail_gate,
                                                            int32_t* __restrict__ seq_len) {
    const int b = blockIdx.x, tid = threadIdx.x;
    const uint16_t* rb = raw + (size_t)b * T * kDim;
    // window: tokens max(0, T-W) .. T-1; thread handles 4 dims (8 bytes of bf16)
    const int64_t w0 = max64(0, T - W);
    for (int64_t t = w0; t < T; ++t) {
        const uint2 x = *reinterpret_cast<const uint2*>(rb + (size_t)t * kDim + 4 * tid);
        uint8_t* e = win_kv + ((size_t)b * W + (size_t)(t % W)) * kEntry;
        if (tid < kNope / 4) {
            const uint32_t v = f32_to_e4m3(bf16_bits_to_f32(x.x)) | (f32_to_e4m3(bf16_bits_to_f32(x.x >> 16)) << 8) |
                               (f32_to_e4m3(bf16_bits_to_f32(x.y)) << 16) |
                               (f32_to_e4m3(bf16_bits_to_f32(x.y >> 16)) << 24);
            *reinterpret_cast<uint32_t*>(e + 4 * tid) = v;
        } else {
            *reinterpret_cast<uint2*>(e + kNope + 8 * (tid - kNope / 4)) = x;
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
                                 int32_t* seq_len, cudaStream_t stream) {
    prefill_state_kernel<<<B, 128, 0, stream>>>(raw, gate, T, m, W, win_kv, tail_kv, tail_gate, seq_len);
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

__global__ void __launch_bounds__(kAppendThreads) append_kernel(csld_layer_cache cache,
                                                                const uint16_t* __restrict__ kv_new,
                                                                const float* __restrict__ gate_new,
                                                                int32_t* err) {
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
            const uint32_t v = f32_to_e4m3(bf16_bits_to_f32(x.x)) |
                               (f32_to_e4m3(bf16_bits_to_f32(x.x >> 16)) << 8) |
                               (f32_to_e4m3(bf16_bits_to_f32(x.y)) << 16) |
                               (f32_to_e4m3(bf16_bits_to_f32(x.y >> 16)) << 24);
            *reinterpret_cast<uint32_t*>(e + 4 * tid) = v;
        } else {
            *reinterpret_cast<uint2*>(e + kNope + 8 * (tid - kNope / 4)) = x;
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
            warp_store_entry(cache.comp_kv + ((size_t)b * cap + (size_t)s) * kEntry, lane, c);
#pragma unroll
            for (int d = 0; d < 16; ++d) cbuf[16 * lane + d] = bf16_bits_to_f32(f32_to_bf16_bits(c[d]));
        }
        if (cache.has_indexer) {
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
                          const float* gate_new, int32_t* err, cudaStream_t stream) {
    cudaError_t e = launch_pdl(append_kernel, dim3(cache.batch), dim3(kAppendThreads), 0, stream, cache, kv_new, gate_new, err);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace csld
