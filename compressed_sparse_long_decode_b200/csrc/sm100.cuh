// Blackwell (sm_100a) tensor-memory, 5th-generation tensor-core and tensor-copy helpers.
// Internal to libcsld.
//
// Conventions used by the callers:
//  * TMEM addresses are (lane << 16) | column.  A warp may only touch the 32 lanes of its
//    sub-partition: lanes 32*(warp % 4) .. 32*(warp % 4) + 31.
//  * tcgen05.mma / tcgen05.commit are issued by one thread; tcgen05.alloc / dealloc / ld / st
//    are warp-collective (.sync.aligned).
//  * The indexer's shared-memory operands use the K-major, 32-byte-swizzle canonical layout:
//    rows of 32 bytes, 8-row groups of 256 bytes, and inside every group the two 16-byte
//    halves of rows 4..7 exchanged (byte-address bit 4 XOR bit 7).  The key cache is stored
//    that way, so bulk copies reproduce it; hand-written operands apply the same XOR.  The
//    attention's operands use the 128-byte swizzle that its tensor maps write.
#pragma once
#include <cuda.h>
#include <stdint.h>

#include "csld_internal.cuh"

namespace csld {

// ---- tensor memory ------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(smem_u32(slot)), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(taddr), "r"(ncols) : "memory");
}
// Order tcgen05 operations around thread synchronisation (barriers, mbarrier waits).
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Make this thread's ordinary shared-memory writes visible to the tensor cores / TMA.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 32 lanes x 16 columns of 32 bits: thread i gets lane (base lane + i), columns col .. col+15.
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
// Writes v to 8 consecutive columns of the warp's 32 lanes.
__device__ __forceinline__ void tmem_st_32x32b_x8_fill(uint32_t taddr, uint32_t v) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %1, %1, %1, %1, %1, %1, %1};"
                 :: "r"(taddr), "r"(v) : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ---- shared-memory matrix descriptor --------------------------------------------------------
// K-major operand in the 32-byte-swizzle layout starting at p (256-byte aligned): rows of 32
// bytes, 8-row groups 256 bytes apart.  Fields: start address >> 4 (bits 0-13), leading byte
// offset >> 4 (16-29; unused by swizzled K-major layouts whose K fits one row), stride byte
// offset >> 4 (32-45), descriptor version 1 (46-47), base offset 0, swizzle mode 6 = 32 B
// (61-63).
__device__ __forceinline__ uint64_t smem_desc_kmajor_sw32(const void* p) {
    const uint32_t a = smem_u32(p);
    uint64_t d = static_cast<uint64_t>((a >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>(1u) << 16;
    d |= static_cast<uint64_t>(256u >> 4) << 32;
    d |= static_cast<uint64_t>(1u) << 46;
    d |= static_cast<uint64_t>(6u) << 61;
    return d;
}

// Instruction descriptor of the block-scaled FP4 MMA (kind::mxf4): A and B E2M1 (format 1),
// K-major, UE8M0 scale factors (bit 23), N = n (bits 17-22 hold n / 8), M = 128 (bits 24-28
// hold M / 16), scale-factor byte selectors 0, dense, K = 64 per instruction.
__host__ __device__ constexpr uint32_t idesc_mxf4_m128(uint32_t n) {
    return (1u << 7) | (1u << 10) | ((n >> 3) << 17) | (1u << 23) | ((128u >> 4) << 24);
}

// D[tmem] (=|+=) A x B^T, A 128 x 64 E2M1 and B n x 64 E2M1 from shared memory, each 32-element
// K block scaled by its UE8M0 factor from TMEM (sfa, sfb), fp32 accumulate.
__device__ __forceinline__ void umma_mxf4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
        :: "r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}
// Arrive once on the mbarrier when every tcgen05.mma issued so far by this thread completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 :: "r"(smem_u32(bar)) : "memory");
}

// ---- tensor maps -------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_map(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" :: "l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void tmem_st_32x32b_x1(uint32_t taddr, uint32_t v) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" :: "r"(taddr), "r"(v) : "memory");
}

// Instruction descriptors (M = 128, fp32 accumulation):
//  kind::f8f6f4  E4M3 x E4M3: c fp32 (bit 4), a/b format 0, majors in bits 15/16, N/8 in
//  bits 17-22, M/16 in 24-28.
__host__ __device__ constexpr uint32_t idesc_e4m3_m128(uint32_t n, bool a_mn, bool b_mn) {
    return (1u << 4) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) | ((n >> 3) << 17) | ((128u >> 4) << 24);
}
//  kind::f16  BF16 x BF16 (a/b format 1).
__host__ __device__ constexpr uint32_t idesc_bf16_m128(uint32_t n, bool a_mn, bool b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
           ((n >> 3) << 17) | ((128u >> 4) << 24);
}
//  kind::mxf8f6f4 block-scaled E4M3 x E4M3, UE8M0 scales (bit 23), B scale byte in bits 4-5.
__host__ __device__ constexpr uint32_t idesc_mxe4m3_m128(uint32_t n, bool a_mn, bool b_mn, uint32_t b_sf_id) {
    return ((b_sf_id & 3u) << 4) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) | ((n >> 3) << 17) |
           (1u << 23) | ((128u >> 4) << 24);
}

__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n\t}"
        :: "r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0u) : "memory");
}
__device__ __forceinline__ void umma_f8f6f4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n\t}"
        :: "r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0u) : "memory");
}
// Block-scaled 8-bit MMA: each 32-element K block scaled by UE8M0 factors read from TMEM (the
// byte selected by bits 30-31 of the scale addresses, which must match the ids in idesc).
__device__ __forceinline__ void umma_mxf8f6f4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                              uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
        :: "r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}

__device__ __forceinline__ void tmem_ld_32x32b_x8(uint32_t taddr, uint32_t (&r)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
}
__device__ __forceinline__ void tmem_st_32x32b_x8(uint32_t taddr, const uint32_t (&r)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};"
                 :: "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
                 : "memory");
}

// Offset of byte c of row r in a [rows][128 B] block with the 128-byte swizzle (the 16-byte
// chunk index XOR the row index within each 8-row, 1024-byte atom).
__device__ __forceinline__ int sw128(int r, int c) {
    return (r >> 3) * 1024 + (r & 7) * 128 + ((((c >> 4) ^ r) & 7) << 4) + (c & 15);
}
// Operand with the 128-byte swizzle (1024-byte aligned atoms): 8-row groups 1024 bytes apart
// (SBO); LBO = stride between 128-byte column blocks of an MN-major operand wider than 128 B.
// Advancing the start address by 32 bytes inside the row selects the next K slice of a K-major
// operand.
__device__ __forceinline__ uint64_t desc_sw128(const void* p, uint32_t lbo) {
    const uint32_t a = smem_u32(p);
    uint64_t d = static_cast<uint64_t>((a >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>(1024u >> 4) << 32;
    d |= static_cast<uint64_t>(1u) << 46;
    d |= static_cast<uint64_t>(2u) << 61;
    return d;
}

// 2-D tensor map over a byte array of `rows` rows of `row_bytes` bytes (row_bytes a multiple of
// 16, base 16-byte aligned): boxes of box_x bytes (<= 128) by box_y rows, 128-byte swizzle in
// shared memory, rows past the end read as zeros.  Host only.  Returns false on failure.
bool make_tensor_map_2d_u8(CUtensorMap* map, const void* base, uint64_t row_bytes, uint64_t rows, uint32_t box_x,
                           uint32_t box_y);

}  // namespace csld
