// Hybrid decode attention over FP8/bf16 compressed entries plus a sliding window.
//
// Source: "DeepSeek-V4: a million-token context that agents can actually use" -- CSA paragraph
// and Figure 3 caption (each query attends to its top-k compressed blocks; a sliding-window
// branch covers the most recent uncompressed tokens), HCA paragraph and Figure 4 caption
// (every query attends densely to all compressed blocks; the same window branch), storage
// paragraph (entries FP8 except the RoPE dims in bf16); velog.io paper review, core
// techniques 1-2.  Keys and values are the same decoded 512-d entry (one KV head); 16 query
// heads share it; one softmax runs over {selected or all visible entries} + {window tokens}.
//
// Two kernels: attention_tc_partial_kernel (attention_tc.cu) runs each split of each
// sequence's key list on the tensor cores and leaves the split's unnormalised O, its running max
// m (log2 units) and its sum l in the workspace; attention_merge_kernel below combines the
// splits with log-sum-exp weights into out and lse.  This file also holds the split plan and the
// library-owned scratch of the allocation-free entry point.
#include <mutex>

#include "csld_internal.cuh"
#include "kernels.cuh"

namespace csld {

// Merge the splits of one (sequence, head): out = sum_j 2^(m_j - M) O_j / L,
// lse = ln 2 * (M + log2 L) with L = sum_j 2^(m_j - M) l_j over the non-empty splits (M = their
// largest m).  512 threads: thread t owns dims 4 (t % 128) .. +3 and adds every fourth split
// starting at t / 128; the four partial sums are then added in a fixed order.  Every thread
// issues its O loads before warp 0 forms the split weights, so the merge costs about one round
// trip to L2.  kv_scale (scaled FP8 entries; 1 for the base layout): the partials' FP8 dims
// (0..447) are in units of the entries' codes and are multiplied by it here.
constexpr int kMergeThreads = 512;
constexpr int kMergeGroups = kMergeThreads / (kDim / 4);   // 4
constexpr int kMergeU = 8;                                 // O loads a thread keeps in flight
__global__ void __launch_bounds__(kMergeThreads) attention_merge_kernel(const float* __restrict__ opart,
                                                                        const float2* __restrict__ mlpart,
                                                                        int splits, float* __restrict__ out,
                                                                        float* __restrict__ lse_out, float kv_scale) {
    __shared__ float fw[256];
    __shared__ float4 red[kMergeGroups - 1][kDim / 4];
    __shared__ float mlw[2];
    const int b = blockIdx.x, h = blockIdx.y, tid = threadIdx.x, lane = tid & 31;
    const int d4 = tid % (kDim / 4), g = tid / (kDim / 4);
    pdl_wait();      // the partials come from the partial kernel
    pdl_trigger();
    const int ns = min(splits, 256);
    const float4* ob = reinterpret_cast<const float4*>(opart + ((size_t)b * splits * kHeads + h) * kDim) + d4;
    const size_t jstride = (size_t)kHeads * kDim / 4;
    float4 v[kMergeU];
#pragma unroll
    for (int u = 0; u < kMergeU; ++u) {
        const int j = g + kMergeGroups * u;
        v[u] = j < ns ? __ldcg(ob + (size_t)j * jstride) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if (tid < 32) {
        float2 ml[8];
        float M = -INFINITY;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int j = lane + 32 * i;
            ml[i] = j < ns ? __ldcg(&mlpart[((size_t)b * splits + j) * kHeads + h]) : make_float2(-INFINITY, 0.f);
            if (ml[i].y > 0.f) M = fmaxf(M, ml[i].x);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        float Lp = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int j = lane + 32 * i;
            const float f = (ml[i].y > 0.f && M != -INFINITY) ? exp2f(ml[i].x - M) : 0.f;
            if (j < ns) fw[j] = f;
            Lp += f * ml[i].y;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) Lp += __shfl_xor_sync(0xffffffffu, Lp, o);
        if (lane == 0) {
            mlw[0] = M;
            mlw[1] = Lp;
        }
    }
    __syncthreads();
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    auto add = [&](float f, const float4& x) {
        acc.x = fmaf(f, x.x, acc.x);
        acc.y = fmaf(f, x.y, acc.y);
        acc.z = fmaf(f, x.z, acc.z);
        acc.w = fmaf(f, x.w, acc.w);
    };
#pragma unroll
    for (int u = 0; u < kMergeU; ++u) {
        const int j = g + kMergeGroups * u;
        if (j < ns && fw[j] > 0.f) add(fw[j], v[u]);   // empty splits may hold stale rows
    }
    for (int j = g + kMergeGroups * kMergeU; j < ns; j += kMergeGroups)
        if (fw[j] > 0.f) add(fw[j], __ldcg(ob + (size_t)j * jstride));
    if (g > 0) red[g - 1][d4] = acc;
    __syncthreads();
    if (g == 0) {
#pragma unroll
        for (int gg = 0; gg < kMergeGroups - 1; ++gg) {
            acc.x += red[gg][d4].x;
            acc.y += red[gg][d4].y;
            acc.z += red[gg][d4].z;
            acc.w += red[gg][d4].w;
        }
        const float M = mlw[0], Lsum = mlw[1];
        if (Lsum > 0.f) {
            const float inv = (4 * d4 < kNope) ? (1.f / Lsum) * kv_scale : 1.f / Lsum;
            acc.x *= inv;
            acc.y *= inv;
            acc.z *= inv;
            acc.w *= inv;
        }
        reinterpret_cast<float4*>(out + ((size_t)b * kHeads + h) * kDim)[d4] = acc;
        if (lse_out && tid == 0)
            lse_out[(size_t)b * kHeads + h] =
                (M == -INFINITY || !(Lsum > 0.f)) ? -INFINITY : (M + log2f(Lsum)) * 0.69314718055994531f;
    }
}

AttentionPlan attention_plan(int B, int64_t cap, int k, bool sparse, int W, int num_sms) {
    AttentionPlan p;
    const int64_t L = (sparse ? (int64_t)k : cap) + W;
    const int64_t tiles = (L + attention_tc_tile() - 1) / attention_tc_tile();
    int64_t s = num_sms / (B > 0 ? B : 1);
    if (s < 1) s = 1;
    if (s > tiles) s = tiles;
    if (s < 1) s = 1;
    if (s > 256) s = 256;   // the merge kernel handles up to 256 splits
    p.splits = static_cast<int>(s);
    p.ws_bytes = (size_t)B * p.splits * kHeads * (kDim * sizeof(float) + sizeof(float2));
    return p;
}

cudaError_t launch_attention(const uint16_t* q, const uint8_t* comp_kv, int64_t cap, int ratio,
                             const int32_t* topk, int k, const uint8_t* win_kv, int W, int Wr, int Q,
                             const int32_t* seq_len, int B, float scale, float* out,
                             float* lse_out, void* ws, const AttentionPlan& plan, int32_t* err,
                             cudaStream_t stream, float kv_scale) {
    // B cache rows, Q query rows each: the plan and the partials count B * Q query rows
    float* opart = static_cast<float*>(ws);
    float2* mlpart = reinterpret_cast<float2*>(opart + (size_t)B * Q * plan.splits * kHeads * kDim);
    cudaError_t e = launch_attention_tc_partial(q, comp_kv, cap, ratio, topk, k, win_kv, W, Wr, Q, seq_len, B, scale,
                                                plan.splits, opart, mlpart, err, stream, kv_scale);
    if (e != cudaSuccess) return e;
    e = launch_pdl(attention_merge_kernel, dim3(B * Q, kHeads), dim3(kMergeThreads), 0, stream,
                   static_cast<const float*>(opart), static_cast<const float2*>(mlpart), plan.splits, out, lse_out,
                   kv_scale);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------
// Library-owned scratch for callers that cannot allocate device memory (see
// hybrid_decode_attention_static in csld.h).  The array lives in the library's module: every
// GPU that loads the library holds these bytes until the process exits.  Host code must not
// hand the array's name to a kernel (on the host it only stands for the symbol); the device
// address is looked up once per device with cudaGetSymbolAddress.
// ------------------------------------------------------------------------------------------
static __device__ __align__(256) uint8_t g_attention_static_scratch[CSLD_STATIC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_static_mu;
void* g_static_ptr[kMaxDevices] = {};
}  // namespace

cudaError_t attention_static_scratch(void** ptr) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_static_mu);
    if (g_static_ptr[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_attention_static_scratch);   // the current device's copy
        if (e != cudaSuccess) return e;
        g_static_ptr[dev] = p;
    }
    *ptr = g_static_ptr[dev];
    return cudaSuccess;
}

}  // namespace csld
