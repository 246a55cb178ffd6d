// Context-parallel decode: one sequence's compressed cache split into contiguous entry ranges
// held by different GPUs.  The kernels here are the per-rank steps around the two exchanges:
//
//  1. indexer_rescore_kernel -- the fp32 score of each entry a rank's indexer selected, formed
//     exactly as the indexer forms it (FP4 query and key, exact integer group dots, the fixed
//     fp32 operation order), so the candidates of all ranks compare as the single-GPU indexer
//     would compare them;
//  2. topk_merge_kernel -- after the candidates (score, global index) of every rank have been
//     gathered: the exact top-k by (score desc, index asc) over them, written as this rank's
//     local indices (entries outside its range become -1);
//  3. lse_merge_kernel -- after every rank's attention output and log-sum-exp have been
//     gathered: the exact combination out = sum_r exp(lse_r - L) out_r, L = log sum_r exp(lse_r).
//
// Source: "DeepSeek-V4: a million-token context that agents can actually use" -- CSA paragraph
// (the lightning indexer picks the top-k compressed blocks per query), HCA paragraph (dense
// attention over the compressed stream).  The split itself is this library's: the pages run
// everything on one device.  The top-k of a union of ranges is the top-k of the union of each
// range's top-k, and the softmax over a union of key sets is the log-sum-exp combination of the
// softmaxes over its parts, so both merges reproduce the single-GPU result.
#include "csld_internal.cuh"
#include "kernels.cuh"

namespace csld {

namespace {

// Twice the E2M1 value of a 4-bit code as a signed integer (0, +-1, +-2, +-3, +-4, +-6, +-8, +-12).
__device__ __forceinline__ int twice_e2m1(uint32_t code) {
    const uint32_t mag = code & 7u;
    const int v = static_cast<int>(mag < 4u ? ((kTwiceE2M1Lo >> (8u * mag)) & 0xFFu)
                                            : ((kTwiceE2M1Hi >> (8u * (mag - 4u))) & 0xFFu));
    return (code & 8u) ? -v : v;
}

}  // namespace

// One CTA of 128 threads per sequence; thread j scores selected entries j, j + 128, ...
__global__ void __launch_bounds__(128) indexer_rescore_kernel(const uint8_t* __restrict__ ikeys,
                                                              const float* __restrict__ iscales, int64_t cap,
                                                              const float* __restrict__ q_idx,
                                                              const float* __restrict__ head_w,
                                                              const int32_t* __restrict__ sel, int k,
                                                              float* __restrict__ scores) {
    __shared__ int qv[kIdxHeads][kIdxDim];   // twice the FP4 query value (an integer)
    __shared__ float qs[kIdxHeads][2];       // the query's group scales
    const int b = blockIdx.x, tid = threadIdx.x;
    pdl_wait();
    pdl_trigger();
    if (tid < 2 * kIdxHeads) {   // thread (h, g): quantise group g of head h like the keys
        const int h = tid >> 1, g = tid & 1;
        const float* x = q_idx + ((size_t)b * kIdxHeads + h) * kIdxDim + 32 * g;
        float amax = 0.f;
        for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(x[i]));
        const float sg = fp4_group_scale(amax);
        const float inv = 1.0f / sg;   // exact: a power of two
        for (int i = 0; i < 32; ++i) qv[h][32 * g + i] = twice_e2m1(e2m1_code(x[i] * inv));
        qs[h][g] = sg;
    }
    __syncthreads();
    const float w0 = head_w[b * kIdxHeads + 0], w1 = head_w[b * kIdxHeads + 1];
    const float w2 = head_w[b * kIdxHeads + 2], w3 = head_w[b * kIdxHeads + 3];
    for (int j = tid; j < k; j += blockDim.x) {
        const int32_t s = sel[(size_t)b * k + j];
        if (s < 0 || s >= cap) {
            scores[(size_t)b * k + j] = -INFINITY;
            continue;
        }
        // logical byte c of entry s sits at c XOR 16 * bit 2 of s (the stored key layout)
        const uint8_t* kc = ikeys + ((size_t)b * cap + (size_t)s) * kIkey;
        const int swap = static_cast<int>((s >> 2) & 1) * 16;
        const float2 ks = *reinterpret_cast<const float2*>(iscales + ((size_t)b * cap + (size_t)s) * 2);
        int dot[kIdxHeads][2] = {};
        for (int c = 0; c < kIkey; ++c) {
            const uint32_t byte = kc[c ^ swap];
            const int e0 = twice_e2m1(byte & 15u), e1 = twice_e2m1(byte >> 4);
            const int g = c >> 4;
#pragma unroll
            for (int h = 0; h < kIdxHeads; ++h) dot[h][g] += qv[h][2 * c] * e0 + qv[h][2 * c + 1] * e1;
        }
        float rr[kIdxHeads];
#pragma unroll
        for (int h = 0; h < kIdxHeads; ++h) {
            // d = fma(I1, s1, I0*s0) with s_g = (qscale_g * kscale_g) * 0.25
            const float s0 = __fmul_rn(__fmul_rn(qs[h][0], ks.x), 0.25f);
            const float s1 = __fmul_rn(__fmul_rn(qs[h][1], ks.y), 0.25f);
            const float d = __fmaf_rn(static_cast<float>(dot[h][1]), s1, __fmul_rn(static_cast<float>(dot[h][0]), s0));
            rr[h] = d > 0.f ? d : 0.f;
        }
        float sc = __fmul_rn(w0, rr[0]);
        sc = __fmaf_rn(w1, rr[1], sc);
        sc = __fmaf_rn(w2, rr[2], sc);
        sc = __fmaf_rn(w3, rr[3], sc);
        scores[(size_t)b * k + j] = sc;
    }
}

// Exact top-k over the C gathered candidates of one sequence (one CTA of 1024 threads per
// sequence, bitonic sort of 64-bit keys in shared memory: C <= kMergeMaxCand).  Key = score_key
// (order-preserving) << 32 | (2^31 - 1 - global index), so a larger key is a better (score desc,
// index asc) candidate; empty candidates (index < 0) get key 0.  The k best are written as
// indices local to [lo, lo + n_local) in ascending order (others -1), padded with -1.
constexpr int kMergeMaxCand = 16384;
__global__ void __launch_bounds__(1024) topk_merge_kernel(const float* __restrict__ cand_score,
                                                          const int32_t* __restrict__ cand_idx,
                                                          const int64_t* __restrict__ rank_lo, int R, int k,
                                                          int64_t lo, int64_t n_local, int32_t* __restrict__ out) {
    extern __shared__ __align__(16) uint64_t key[];
    const int b = blockIdx.x, tid = threadIdx.x;
    const int C = R * k;
    int P = 1;
    while (P < C) P <<= 1;
    pdl_wait();
    pdl_trigger();
    // candidates of sequence b: rank r's row b holds k of them ([R][B][k] layout), as indices
    // local to the rank's range, which starts at rank_lo[r]
    for (int i = tid; i < P; i += blockDim.x) {
        uint64_t v = 0ull;
        if (i < C) {
            const int r = i / k, j = i % k;
            const size_t at = ((size_t)r * gridDim.x + b) * k + j;
            const int32_t li = cand_idx[at];
            const int64_t g = li < 0 ? -1 : rank_lo[r] + li;
            if (g >= 0 && g < 0x7FFFFFFF)
                v = (static_cast<uint64_t>(score_key(cand_score[at])) << 32) | (0x7FFFFFFFu - static_cast<uint32_t>(g));
        }
        key[i] = v;
    }
    __syncthreads();
    // bitonic sort, descending
    for (int size = 2; size <= P; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int i = tid; i < P; i += blockDim.x) {
                const int j = i ^ stride;
                if (j > i) {
                    const bool desc = (i & size) == 0;
                    const uint64_t a = key[i], c = key[j];
                    if ((a < c) == desc) {
                        key[i] = c;
                        key[j] = a;
                    }
                }
            }
            __syncthreads();
        }
    }
    // the k best (fewer if there are fewer candidates), as global indices, then ascending
    const int take = k < P ? k : P;
    for (int i = tid; i < take; i += blockDim.x) {
        const uint64_t v = key[i];
        key[i] = v ? static_cast<uint64_t>(0x7FFFFFFFu - static_cast<uint32_t>(v & 0xFFFFFFFFu)) : 0xFFFFFFFFull;
    }
    for (int i = take + tid; i < P; i += blockDim.x) key[i] = 0xFFFFFFFFull;
    __syncthreads();
    for (int size = 2; size <= P; size <<= 1) {   // ascending
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int i = tid; i < P; i += blockDim.x) {
                const int j = i ^ stride;
                if (j > i) {
                    const bool asc = (i & size) == 0;
                    const uint64_t a = key[i], c = key[j];
                    if ((a > c) == asc) {
                        key[i] = c;
                        key[j] = a;
                    }
                }
            }
            __syncthreads();
        }
    }
    for (int i = tid; i < k; i += blockDim.x) {
        int32_t v = -1;
        if (i < take && key[i] != 0xFFFFFFFFull) {
            const int64_t g = static_cast<int64_t>(key[i]);
            if (g >= lo && g < lo + n_local) v = static_cast<int32_t>(g - lo);
        }
        out[(size_t)b * k + i] = v;
    }
}

// out[b][h] = sum_r exp(lse_r - L) out_r[b][h],  L = log sum_r exp(lse_r) (natural log); ranks
// with lse = -inf (an empty key set) contribute nothing.  One CTA of 128 threads per (b, h).
__global__ void __launch_bounds__(128) lse_merge_kernel(const float* __restrict__ outs, const float* __restrict__ lses,
                                                        int R, int BH, float* __restrict__ out,
                                                        float* __restrict__ lse) {
    const int bh = blockIdx.x, tid = threadIdx.x;
    pdl_wait();
    pdl_trigger();
    float M = -INFINITY;
    for (int r = 0; r < R; ++r) M = fmaxf(M, lses[(size_t)r * BH + bh]);
    float L = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (M != -INFINITY) {
        for (int r = 0; r < R; ++r) {
            const float l = lses[(size_t)r * BH + bh];
            if (l == -INFINITY) continue;
            const float w = expf(l - M);
            L += w;
            const float4 v = reinterpret_cast<const float4*>(outs + ((size_t)r * BH + bh) * kDim)[tid];
            acc.x = fmaf(w, v.x, acc.x);
            acc.y = fmaf(w, v.y, acc.y);
            acc.z = fmaf(w, v.z, acc.z);
            acc.w = fmaf(w, v.w, acc.w);
        }
        const float inv = 1.f / L;
        acc.x *= inv;
        acc.y *= inv;
        acc.z *= inv;
        acc.w *= inv;
    }
    reinterpret_cast<float4*>(out + (size_t)bh * kDim)[tid] = acc;
    if (lse && tid == 0) lse[bh] = (M == -INFINITY) ? -INFINITY : M + logf(L);
}

cudaError_t launch_indexer_rescore(const uint8_t* ikeys, const float* iscales, int64_t cap, const float* q_idx,
                                   const float* head_w, const int32_t* sel, int B, int k, float* scores,
                                   cudaStream_t stream) {
    cudaError_t e = launch_pdl(indexer_rescore_kernel, dim3(B), dim3(128), 0, stream, ikeys, iscales, cap, q_idx,
                               head_w, sel, k, scores);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

int topk_merge_max_candidates() { return kMergeMaxCand; }

cudaError_t launch_topk_merge(const float* cand_score, const int32_t* cand_idx, const int64_t* rank_lo, int R, int B,
                              int k, int64_t lo, int64_t n_local, int32_t* out, cudaStream_t stream) {
    int P = 1;
    while (P < R * k) P <<= 1;
    const size_t smem = (size_t)P * sizeof(uint64_t);
    cudaError_t e = set_smem_once(topk_merge_kernel, (size_t)kMergeMaxCand * sizeof(uint64_t));
    if (e != cudaSuccess) return e;
    e = launch_pdl(topk_merge_kernel, dim3(B), dim3(1024), smem, stream, cand_score, cand_idx, rank_lo, R, k, lo,
                   n_local, out);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t launch_lse_merge(const float* outs, const float* lses, int R, int BH, float* out, float* lse,
                             cudaStream_t stream) {
    cudaError_t e = launch_pdl(lse_merge_kernel, dim3(BH), dim3(kDim / 4), 0, stream, outs, lses, R, BH, out, lse);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace csld
