// Staging copies by a kernel: between any two device-accessible buffers, i.e. device memory or
// pinned host memory mapped into the device's address space (unified addressing).  A decode
// step's inputs come from the host this way: a kernel node chains to the decode kernel after it
// (and may launch behind the kernel before it), where a copy-engine transfer placed between
// two kernels costs a round trip through the copy engine on the step's critical path.
#include "csld_internal.cuh"

namespace csld {

constexpr int kStageThreads = 256;
constexpr int kStageUnroll = 4;

// dst[i] = src[i] for i < n16 (16-byte units).  Each thread loads its first kStageUnroll units
// before waiting for the kernel before this one (which may still read dst; src is not written
// by it), so the reads' latency overlaps that kernel's tail.
__global__ void __launch_bounds__(kStageThreads) stage_kernel(uint4* __restrict__ dst, const uint4* __restrict__ src,
                                                             size_t n16) {
    const size_t stride = (size_t)gridDim.x * kStageThreads;
    size_t i = (size_t)blockIdx.x * kStageThreads + threadIdx.x;
    uint4 v[kStageUnroll];
#pragma unroll
    for (int u = 0; u < kStageUnroll; ++u)
        if (i + u * stride < n16) v[u] = src[i + u * stride];
    pdl_wait();
    pdl_trigger();
#pragma unroll
    for (int u = 0; u < kStageUnroll; ++u)
        if (i + u * stride < n16) dst[i + u * stride] = v[u];
    for (i += kStageUnroll * stride; i < n16; i += stride) dst[i] = src[i];
}

cudaError_t launch_stage(void* dst, const void* src, size_t bytes, int num_sms, cudaStream_t stream) {
    const size_t n16 = bytes / 16;
    if (n16 == 0) return cudaSuccess;
    size_t blocks = (n16 + (size_t)kStageThreads * kStageUnroll - 1) / ((size_t)kStageThreads * kStageUnroll);
    const size_t most = (size_t)num_sms * 8;
    if (blocks > most) blocks = most;
    cudaError_t e = launch_pdl(stage_kernel, dim3(static_cast<unsigned>(blocks)), dim3(kStageThreads), 0, stream,
                               static_cast<uint4*>(dst), static_cast<const uint4*>(src), n16);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace csld
