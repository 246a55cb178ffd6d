// Internal device helpers of libcsld (sm_100a).  Not part of the ABI.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "csld.h"

namespace csld {

__host__ __device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }
__host__ __device__ __forceinline__ int64_t max64(int64_t a, int64_t b) { return a > b ? a : b; }

constexpr int kDim = CSLD_DIM;
constexpr int kNope = CSLD_DIM_NOPE;
constexpr int kRope = CSLD_DIM_ROPE;
constexpr int kEntry = CSLD_ENTRY_BYTES;
constexpr int kHeads = CSLD_HEADS;
constexpr int kIdxHeads = CSLD_IDX_HEADS;
constexpr int kIdxDim = CSLD_IDX_DIM;
constexpr int kIkey = CSLD_IKEY_BYTES;

// ------------------------------------------------------------------------------------------
// Shared-memory addressing, mbarriers and bulk (TMA) copies.
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

// Make initialised barriers visible to the async (bulk-copy) proxy.
__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait on an mbarrier phase: polls first (try_wait itself suspends briefly), then
// backs off with short sleeps.  Returns false if the phase did not complete within about a
// second; callers then record CSLD_DEVERR_TIMEOUT and stop issuing work.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
    for (uint32_t i = 0; i < (1u << 22); ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if (i >= 32) __nanosleep(128);
    }
    return false;
}

// 1-D bulk copy global -> shared, completing `bytes` on the mbarrier.  src, dst 16-byte
// aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void named_barrier(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
// Named barrier that also ORs a predicate over its threads: every thread gets the same answer,
// so a group can leave a loop together when any of its threads saw a failed wait.
__device__ __forceinline__ bool named_barrier_or(int id, int nthreads, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, %2, %3, p;\n selp.u32 %0, 1, 0, q;\n}"
        : "=r"(r)
        : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3,
                                            const void* p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(smem_u32(p)));
}

// ------------------------------------------------------------------------------------------
// Number formats.  E4M3 / bf16 conversions use the hardware round-to-nearest-even converts;
// E2M1 (FP4) is written out below from the grid {0, .5, 1, 1.5, 2, 3, 4, 6}.
// ------------------------------------------------------------------------------------------
// Two E4M3 bytes (low byte = first element) -> f16x2 (low half = first element); exact.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two_bytes) {
    uint32_t r;
    asm("{\n .reg .b16 t;\n cvt.u16.u32 t, %1;\n cvt.rn.f16x2.e4m3x2 %0, t;\n}\n"
        : "=r"(r)
        : "r"(two_bytes));
    return r;
}

// Four E4M3 bytes -> two f16x2 (bytes 0,1 -> lo; bytes 2,3 -> hi); exact.  The 32-bit word
// is split into its 16-bit halves in place, so each pair costs one convert.
__device__ __forceinline__ void e4m3x4_to_f16x2x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
    asm("{\n .reg .b16 l, h;\n mov.b32 {l, h}, %2;\n cvt.rn.f16x2.e4m3x2 %0, l;\n"
        " cvt.rn.f16x2.e4m3x2 %1, h;\n}\n"
        : "=r"(lo), "=r"(hi)
        : "r"(w));
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// E4M3 byte -> fp32 (exact).
__device__ __forceinline__ float e4m3_to_f32(uint32_t byte) {
    uint32_t h2, dummy;
    e4m3x4_to_f16x2x2(byte & 0xFFu, h2, dummy);
    return __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
}

// fp32 -> E4M3 byte: round to nearest even, saturating to +-448.
__device__ __forceinline__ uint32_t f32_to_e4m3(float x) {
    return static_cast<uint32_t>(__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3));
}

__device__ __forceinline__ uint32_t f32_to_bf16_bits(float x) {
    return static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(x)));
}

// (a, b) -> bf16 bits (low half = a), round to nearest even.
__device__ __forceinline__ uint32_t f32x2_to_bf16x2_bits(float a, float b) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&v);
}

// 2^x by the hardware approximation with subnormal results flushed to zero (ex2.approx.ftz).
// Used for softmax weights relative to a running maximum, where anything below 2^-126 is
// negligible; 2^-inf = +0.
__device__ __forceinline__ float exp2_ftz(float x) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t h) {
    return __uint_as_float((h & 0xFFFFu) << 16);
}

// E2M1 code of v (|v| <= 6 expected; larger saturates): nearest grid value, ties to the even
// mantissa (0.25->0, 0.75->1, 1.25->1, 1.75->2, 2.5->2, 3.5->4, 5->4).  Bit 3 = sign.
// Branch-free: the magnitude index is the number of midpoints between grid values that lie
// below |v|, a midpoint counting when |v| is past it (strictly, where the even index is below
// it; from the midpoint on, where the even index is above it); NaN gives 7, as the branch
// chain it replaces did for every input.  A chain of branches here diverges across the lanes of
// a warp (every lane holds a different value) and serialises the FP4 quantisation of the keys.
__device__ __forceinline__ uint32_t e2m1_code(float v) {
    const float a = fabsf(v);
    const uint32_t m = static_cast<uint32_t>(a > 0.25f) + static_cast<uint32_t>(a >= 0.75f) +
                       static_cast<uint32_t>(a > 1.25f) + static_cast<uint32_t>(a >= 1.75f) +
                       static_cast<uint32_t>(a > 2.5f) + static_cast<uint32_t>(a >= 3.5f) +
                       static_cast<uint32_t>(a > 5.0f);
    return (signbit(v) ? 8u : 0u) | (a != a ? 7u : m);
}

// Twice the value of an E2M1 magnitude index 0..7 (an integer): 0,1,2,3,4,6,8,12.
constexpr uint32_t kTwiceE2M1Lo = 0x03020100u;  // indices 0..3
constexpr uint32_t kTwiceE2M1Hi = 0x0C080604u;  // indices 4..7

// Smallest power of two sigma with amax <= 6*sigma; 1 when amax == 0.  Exact: with
// 2^e0 <= amax < 2^(e0+1), sigma is 2^(e0-2) if amax <= 1.5*2^e0, else 2^(e0-1).
__device__ __forceinline__ float fp4_group_scale(float amax) {
    if (!(amax > 0.f)) return 1.f;
    const int e0 = ilogbf(amax);
    return (amax <= ldexpf(1.5f, e0)) ? ldexpf(1.f, e0 - 2) : ldexpf(1.f, e0 - 1);
}

// Order-preserving 32-bit key of an fp32 score (-0 and +0 map to the same key).
__device__ __forceinline__ uint32_t score_key(float s) {
    uint32_t u = __float_as_uint(s);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Programmatic dependent launch.  A kernel launched with launch_pdl may start while the
// kernel before it in the stream is still running; pdl_wait() blocks until that kernel has
// completed and its memory is visible, so every read of data produced upstream must follow it.
// pdl_trigger() lets the next kernel start launching; it is issued only after pdl_wait(), so
// anything upstream of this kernel is complete by then.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

// Opt a kernel into its dynamic shared-memory size, once per (kernel, device): a function
// attribute, not a stream operation, so later calls may be captured into CUDA graphs.  The
// record is keyed by the kernel's address and the current device, so every GPU a process drives
// gets the attribute set before its first launch there.
cudaError_t set_smem_attr_once(const void* kernel, size_t bytes);
template <typename K>
inline cudaError_t set_smem_once(K kernel, size_t bytes) {
    return set_smem_attr_once(reinterpret_cast<const void*>(kernel), bytes);
}

__device__ __forceinline__ void dev_error(int32_t* err, uint32_t flag) {
    if (err) atomicOr(reinterpret_cast<unsigned int*>(err), flag);
}

}  // namespace csld
