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
// lse = ln 2 * (M + log2 L) with L = sum_j 2^(m_j - M) l_j.  The split summaries go through
// shared memory; the O rows are read 8 splits at a time so their loads overlap.
__global__ void __launch_bounds__(128) attention_merge_kernel(const float* __restrict__ opart,
                                                              const float2* __restrict__ mlpart,
                                                              int splits, float* __restrict__ out,
                                                              float* __restrict__ lse_out) {
    __shared__ float fsh[256];
    __shared__ float lw[4];
    const int b = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
    pdl_wait();      // the partials come from the partial kernel
    pdl_trigger();
    const int ns = min(splits, 256);
    // 1) summaries: M = max over non-empty splits, f_j = 2^(m_j - M), L = sum f_j l_j
    float mj[2], lj[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int j = tid + 128 * r;
        const float2 ml = j < ns ? mlpart[((size_t)b * splits + j) * kHeads + h] : make_float2(-INFINITY, 0.f);
        mj[r] = ml.y > 0.f ? ml.x : -INFINITY;
        lj[r] = ml.y;
    }
    float M = fmaxf(mj[0], mj[1]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    if ((tid & 31) == 0) fsh[tid >> 5] = M;
    __syncthreads();
    M = fmaxf(fmaxf(fsh[0], fsh[1]), fmaxf(fsh[2], fsh[3]));
    __syncthreads();
    float Lp = 0.f;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int j = tid + 128 * r;
        const float f = (M == -INFINITY || mj[r] == -INFINITY) ? 0.f : exp2f(mj[r] - M);
        if (j < ns) fsh[j] = f;
        Lp += f * lj[r];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) Lp += __shfl_xor_sync(0xffffffffu, Lp, o);
    if ((tid & 31) == 0) lw[tid >> 5] = Lp;
    __syncthreads();
    const float Lsum = (lw[0] + lw[1]) + (lw[2] + lw[3]);
    // 2) weighted sum of the O rows; this thread owns dims 4*tid .. 4*tid+3
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    const float4* ob = reinterpret_cast<const float4*>(opart + ((size_t)b * splits * kHeads + h) * kDim) + tid;
    const size_t jstride = (size_t)kHeads * kDim / 4;
    for (int j0 = 0; j0 < ns; j0 += 8) {
        float4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
            v[u] = (j0 + u < ns && fsh[j0 + u] > 0.f) ? ob[(size_t)(j0 + u) * jstride] : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const float f = (j0 + u < ns) ? fsh[j0 + u] : 0.f;
            acc.x += f * v[u].x;
            acc.y += f * v[u].y;
            acc.z += f * v[u].z;
            acc.w += f * v[u].w;
        }
    }
    if (Lsum > 0.f) {
        const float inv = 1.f / Lsum;
        acc.x *= inv;
        acc.y *= inv;
        acc.z *= inv;
        acc.w *= inv;
    }
    reinterpret_cast<float4*>(out + ((size_t)b * kHeads + h) * kDim)[tid] = acc;
    if (lse_out && tid == 0)
        lse_out[(size_t)b * kHeads + h] = (M == -INFINITY || !(Lsum > 0.f)) ? -INFINITY : (M + log2f(Lsum)) * 0.69314718055994531f;
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
                             const int32_t* topk, int k, const uint8_t* win_kv, int W,
                             const int32_t* seq_len, int B, float scale, float* out,
                             float* lse_out, void* ws, const AttentionPlan& plan, int32_t* err,
                             cudaStream_t stream) {
    float* opart = static_cast<float*>(ws);
    float2* mlpart = reinterpret_cast<float2*>(opart + (size_t)B * plan.splits * kHeads * kDim);
    cudaError_t e = launch_attention_tc_partial(q, comp_kv, cap, ratio, topk, k, win_kv, W, seq_len, B, scale,
                                                plan.splits, opart, mlpart, err, stream);
    if (e != cudaSuccess) return e;
    e = launch_pdl(attention_merge_kernel, dim3(B, kHeads), dim3(128), 0, stream, static_cast<const float*>(opart),
                   static_cast<const float2*>(mlpart), plan.splits, out, lse_out);
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
