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
// Kernel design (one CTA = one split of one sequence's key list; 8 warps):
//  - The split's key list is walked in tiles of 64 entries, staged in a 4-stage shared-memory
//    ring.  Warp w gathers entries 8w..8w+7 of a tile with 1-D bulk copies of 576 bytes
//    (sparse mode reads the top-k index, prefetched one tile early; dense mode the position;
//    the window part the ring slot) and arrives on the stage's mbarrier with its byte count;
//    empty slots are zero-filled so they contribute exact zeros.  A stage is refilled right
//    after the first barrier of the following tile, when every warp is done with it.
//  - QK (tensor cores, mma.sync m16n8k16, fp32 accumulate): warp w computes the logits of
//    entries 8w..8w+7 for all 16 heads.  The E4M3 dims are widened in registers with
//    cvt.rn.f16x2.e4m3x2 (exact) and multiplied with the query in f16; the query of head h is
//    pre-scaled by a power of two alpha_h so that max|alpha_h q_h| < 2^14 (exact in f16 for
//    the bf16 inputs); the 64 RoPE dims stay bf16 and use the bf16 MMA on the same
//    accumulators.  The query rows are staged once per CTA by bulk copies and converted once
//    per CTA into shared memory.
//  - Online softmax in the log2 domain; per-tile maxima and P go through double-buffered
//    shared memory, so a tile needs two barriers.  P is kept as f16 (E4M3 dims) and bf16
//    (RoPE dims).
//  - PV: warp w owns output dims 64w..64w+63 for all heads; V fragments are read from the
//    staged bytes (pairs of entries per dim), widened, and multiplied with P.
//  - Each split writes unnormalised O, the running max m (log2 units) and the sum l; a second
//    kernel merges the splits (log-sum-exp) into out and lse.
#include <mutex>

#include "csld_internal.cuh"
#include "kernels.cuh"

namespace csld {

constexpr int kWarps = 8;
constexpr int kAttnThreads = 32 * kWarps;
constexpr int kAT = 64;                        // entries per tile (8 per warp)
constexpr int kAStages = 4;
constexpr int kEStride = 592;                  // staged bytes per entry (576 + 16: conflict-free PV reads)
constexpr int kPStride = kAT + 8;              // P row stride in 16-bit elements (144 bytes)
constexpr int kQStride = kDim + 8;             // staged query row stride in bf16 elements (1040 bytes)
constexpr int kQHStride = kNope + 8;           // f16 query row stride in elements (912 bytes)
constexpr float kLog2e = 1.4426950408889634f;

struct AttnSmem {
    uint8_t stage[kAStages][kAT * kEStride];
    uint16_t qs[kHeads * kQStride];
    uint16_t qf16[kHeads][kQHStride];          // alpha_h q_h of the 448 E4M3 dims, f16
    uint16_t qrope[kHeads][kRope];             // alpha_h q_h of the RoPE dims, bf16
    float c2[kHeads];                          // log2-domain logit factor per head
    uint16_t p16[2][kHeads * kPStride];        // P as f16 [head][entry], double-buffered
    uint16_t pbf[2][kHeads * kPStride];        // P as bf16
    float tmax[2][kWarps][kHeads];
    float lsum[kWarps][kHeads];
    uint8_t valid[kAStages][kWarps];           // bit j of [st][w]: slot 8w+j holds an entry
    uint64_t full[kAStages];
    uint64_t qbar;
    int32_t fail;                              // a bounded wait gave up
};

__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
    const __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&h);
}
__device__ __forceinline__ uint32_t pack_bf162(float a, float b) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&h);
}

__global__ void __launch_bounds__(kAttnThreads, 1) attention_partial_kernel(
    const uint16_t* __restrict__ q, const uint8_t* __restrict__ comp_kv, int64_t cap, int ratio,
    const int32_t* __restrict__ topk, int k, const uint8_t* __restrict__ win_kv, int W,
    const int32_t* __restrict__ seq_len, float scale, int splits, float* __restrict__ opart,
    float2* __restrict__ mlpart, int32_t* err) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    AttnSmem& sm = *reinterpret_cast<AttnSmem*>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, cq = lane & 3;
    const int b = blockIdx.y, split = blockIdx.x;

    // ---- the key list of sequence b and this split's tile range ----------------------------
    int32_t n = seq_len[b];
    if (n < 0) {
        if (tid == 0 && split == 0) dev_error(err, CSLD_DEVERR_SEQ_LEN);
        n = 0;
    }
    const int64_t n_vis = min64(n / ratio, cap);
    const bool sparse = topk != nullptr;
    const int64_t n_comp = sparse ? (int64_t)k : n_vis;            // list slots of the compressed part
    const int n_win = W > 0 ? min(W, n) : 0;
    const int64_t L = n_comp + n_win;
    const int64_t n_tiles_all = (L + kAT - 1) / kAT;
    const int64_t t_begin = n_tiles_all * split / splits;
    const int64_t t_end = n_tiles_all * (split + 1) / splits;
    const int n_tiles = static_cast<int>(t_end - t_begin);

    const size_t part = (size_t)b * splits + split;
    if (n_tiles <= 0) {
        if (tid < kHeads) mlpart[part * kHeads + tid] = make_float2(-INFINITY, 0.f);
        return;
    }

    if (tid == 0) {
        for (int s = 0; s < kAStages; ++s) mbar_init(&sm.full[s], kWarps);
        mbar_init(&sm.qbar, 1);
        sm.fail = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (warp == 0) {
        if (lane == 0) mbar_arrive_expect_tx(&sm.qbar, kHeads * kDim * 2);
        __syncwarp();
        if (lane < kHeads)
            bulk_g2s(sm.qs + lane * kQStride, q + ((size_t)b * kHeads + lane) * kDim, kDim * 2, &sm.qbar);
    }

    // ---- gather: warp w fills slots 8w..8w+7 of tile `it` (lanes 0..7, one entry each) -----
    // Everything here is recomputed from the kernel parameters (constant bank) when needed, so
    // the main loop does not hold the gather state in registers.
    auto slot_of = [&](int it) -> int64_t {
        const int64_t tiles = ((sparse ? (int64_t)k : min64(n / ratio, cap)) + (W > 0 ? min(W, n) : 0) + kAT - 1) / kAT;
        return (tiles * blockIdx.x / splits + it) * kAT + 8 * warp + lane;
    };
    // list slot -> source entry (nullptr: empty slot); `pre` is the prefetched top-k index
    auto source = [&](int64_t i, int32_t pre) -> const uint8_t* {
        const int64_t nv = min64(n / ratio, cap);
        const int64_t nc = sparse ? (int64_t)k : nv;
        const int nw = W > 0 ? min(W, n) : 0;
        if (i >= nc + nw) return nullptr;
        if (i < nc) {
            int64_t v = sparse ? (int64_t)pre : i;
            if (sparse && v >= nv) {
                dev_error(err, CSLD_DEVERR_BAD_INDEX);
                v = -1;
            }
            return v >= 0 ? comp_kv + ((size_t)blockIdx.y * cap + (size_t)v) * kEntry : nullptr;
        }
        const int64_t t = (int64_t)n - nw + (i - nc);
        return win_kv + ((size_t)blockIdx.y * W + (size_t)(t % W)) * kEntry;
    };
    auto prefetch_index = [&](int it) -> int32_t {
        const int64_t i = slot_of(it);
        return (sparse && lane < 8 && it < n_tiles && i < k) ? topk[(size_t)blockIdx.y * k + i] : -1;
    };
    auto produce = [&](int it, int32_t pre) {
        const int st = it % kAStages;
        const uint8_t* src = lane < 8 ? source(slot_of(it), pre) : nullptr;
        uint8_t* dst = sm.stage[st] + (8 * warp + lane) * kEStride;
        if (lane < 8 && src == nullptr) {
            uint4* d4 = reinterpret_cast<uint4*>(dst);
            for (int j = 0; j < kEntry / 16; ++j) d4[j] = make_uint4(0u, 0u, 0u, 0u);
        }
        const uint32_t vm = __ballot_sync(0xffffffffu, src != nullptr);
        if (lane == 0) sm.valid[st][warp] = static_cast<uint8_t>(vm);
        __syncwarp();   // zero-fills and the valid byte precede the arrive (release)
        if (lane == 0) mbar_arrive_expect_tx(&sm.full[st], (uint32_t)__popc(vm) * kEntry);
        __syncwarp();
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        if (src != nullptr) bulk_g2s(dst, src, kEntry, &sm.full[st]);
    };
    for (int it = 0; it < min(n_tiles, kAStages - 1); ++it) produce(it, prefetch_index(it));

    if (!mbar_wait(&sm.qbar, 0)) {
        if (lane == 0) dev_error(err, CSLD_DEVERR_TIMEOUT);
        atomicExch(&sm.fail, 1);
    }
    // ---- the query, once per CTA: 16 threads per head, 32 consecutive dims each -----------
    // alpha_h = 2^(14 - e) with max|q_h| < 2^e, so |alpha_h q_h| < 2^14: bf16 values scaled by a
    // power of two are exact in f16 there (components below 2^-24 of that range flush).
    {
        const int h = tid >> 4, d0 = (tid & 15) * 32;
        const uint16_t* row = sm.qs + h * kQStride + d0;
        float x[32];
        float amax = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint4 v = *reinterpret_cast<const uint4*>(row + 8 * i);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                x[8 * i + 2 * j] = bf16_bits_to_f32(w[j]);
                x[8 * i + 2 * j + 1] = bf16_bits_to_f32(w[j] >> 16);
            }
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(x[i]));
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        int e2 = 0;
        if (amax > 0.f) frexpf(amax, &e2);          // amax < 2^e2
        e2 = max(e2, -100);                         // keep alpha finite for tiny queries
        const float alpha = ldexpf(1.f, 14 - e2);   // alpha * amax < 2^14
        if ((tid & 15) == 0) sm.c2[h] = scale * kLog2e / alpha;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int d = d0 + 2 * i;
            if (d < kNope)
                *reinterpret_cast<uint32_t*>(&sm.qf16[h][d]) = pack_half2(alpha * x[2 * i], alpha * x[2 * i + 1]);
            else
                *reinterpret_cast<uint32_t*>(&sm.qrope[h][d - kNope]) = pack_bf162(alpha * x[2 * i], alpha * x[2 * i + 1]);
        }
    }
    __syncthreads();
    // fragments (A operand, 32 k-steps x 4 registers): k-step s < 28 (E4M3 dims): a0/a1 = dims
    // 112*cq + 4s + {0,1} of heads g / g+8, a2/a3 = dims 112*cq + 4s + {2,3} (the key bytes a
    // thread reads: its 112-byte slice).  k-step 28+s' (RoPE): dims 448 + 16*cq + 4s' + ...
    uint32_t qa[32][4];
    const float c2[2] = {sm.c2[g], sm.c2[g + 8]};
#pragma unroll
    for (int s = 0; s < 28; ++s) {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const uint2 v = *reinterpret_cast<const uint2*>(&sm.qf16[g + 8 * r][112 * cq + 4 * s]);
            qa[s][r] = v.x;
            qa[s][2 + r] = v.y;
        }
    }
#pragma unroll
    for (int s = 0; s < 4; ++s) {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const uint2 v = *reinterpret_cast<const uint2*>(&sm.qrope[g + 8 * r][16 * cq + 4 * s]);
            qa[28 + s][r] = v.x;
            qa[28 + s][2 + r] = v.y;
        }
    }

    float m_run[2] = {-INFINITY, -INFINITY};   // heads g, g+8 (identical in every warp)
    float l_run[2] = {0.f, 0.f};               // this thread's share of the row sums
    float o[8][4];                             // O[heads][64 dims of this warp], 8 n-tiles
#pragma unroll
    for (int j = 0; j < 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
    const bool rope_warp = (warp == kWarps - 1);

    int consumed = 0, produced = min(n_tiles, kAStages - 1);
    bool ok = true;
    for (int it = 0; it < n_tiles; ++it) {
        const int st = it % kAStages, pb = it & 1;
        // the top-k indices of the tile produced in this iteration
        const int32_t pre = prefetch_index(it + kAStages - 1);
        if (!mbar_wait(&sm.full[st], (it / kAStages) & 1)) {
            if (lane == 0) dev_error(err, CSLD_DEVERR_TIMEOUT);
            atomicExch(&sm.fail, 1);
        }
        const uint8_t* stg = sm.stage[st];

        // -- QK: entries 8*warp + g; two accumulators (even / odd k-steps) halve the MMA chain --
        float s4[4] = {0.f, 0.f, 0.f, 0.f};
        {
            float t4[4] = {0.f, 0.f, 0.f, 0.f};
            const uint8_t* ent = stg + (8 * warp + g) * kEStride;
#pragma unroll
            for (int i = 0; i < 7; ++i) {
                const uint4 v = *reinterpret_cast<const uint4*>(ent + 112 * cq + 16 * i);
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int s = 4 * i + j;
                    uint32_t b0, b1;
                    e4m3x4_to_f16x2x2(w[j], b0, b1);
                    if (j & 1) mma_f16(t4, qa[s][0], qa[s][1], qa[s][2], qa[s][3], b0, b1);
                    else mma_f16(s4, qa[s][0], qa[s][1], qa[s][2], qa[s][3], b0, b1);
                }
            }
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const uint4 v = *reinterpret_cast<const uint4*>(ent + kNope + 32 * cq + 16 * i);
                mma_bf16(s4, qa[28 + 2 * i][0], qa[28 + 2 * i][1], qa[28 + 2 * i][2], qa[28 + 2 * i][3], v.x, v.y);
                mma_bf16(t4, qa[29 + 2 * i][0], qa[29 + 2 * i][1], qa[29 + 2 * i][2], qa[29 + 2 * i][3], v.z, v.w);
            }
#pragma unroll
            for (int r = 0; r < 4; ++r) s4[r] += t4[r];
        }
        // s4: (head g, entries e0, e0+1), (head g+8, entries e0, e0+1) with e0 = 8w + 2cq
        const int e0 = 8 * warp + 2 * cq;
        const uint32_t vbyte = sm.valid[st][warp];
        const bool v0 = (vbyte >> (2 * cq)) & 1u, v1 = (vbyte >> (2 * cq + 1)) & 1u;
        float x[4];
        x[0] = v0 ? s4[0] * c2[0] : -INFINITY;
        x[1] = v1 ? s4[1] * c2[0] : -INFINITY;
        x[2] = v0 ? s4[2] * c2[1] : -INFINITY;
        x[3] = v1 ? s4[3] * c2[1] : -INFINITY;
        float mx0 = fmaxf(x[0], x[1]), mx1 = fmaxf(x[2], x[3]);
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        if (cq == 0) {
            sm.tmax[pb][warp][g] = mx0;
            sm.tmax[pb][warp][g + 8] = mx1;
        }
        __syncthreads();   // (A) maxima published; every warp is done with tile it-1
        if (sm.fail) {
            ok = false;
            break;
        }
        // refill the stage of tile it-1 with tile it+kAStages-1
        if (produced < n_tiles && produced == it + kAStages - 1) {
            produce(produced, pre);
            ++produced;
        }
        float tm0 = sm.tmax[pb][0][g], tm1 = sm.tmax[pb][0][g + 8];
#pragma unroll
        for (int w = 1; w < kWarps; ++w) {
            tm0 = fmaxf(tm0, sm.tmax[pb][w][g]);
            tm1 = fmaxf(tm1, sm.tmax[pb][w][g + 8]);
        }
        const float mn0 = fmaxf(m_run[0], tm0), mn1 = fmaxf(m_run[1], tm1);
        // a row with no key yet keeps m = -inf; its p's are 0 and nothing is rescaled
        const float corr0 = (mn0 == -INFINITY) ? 1.f : exp2f(m_run[0] - mn0);
        const float corr1 = (mn1 == -INFINITY) ? 1.f : exp2f(m_run[1] - mn1);
        const float p0 = (mn0 == -INFINITY) ? 0.f : exp2f(x[0] - mn0);
        const float p1 = (mn0 == -INFINITY) ? 0.f : exp2f(x[1] - mn0);
        const float p2 = (mn1 == -INFINITY) ? 0.f : exp2f(x[2] - mn1);
        const float p3 = (mn1 == -INFINITY) ? 0.f : exp2f(x[3] - mn1);
        m_run[0] = mn0;
        m_run[1] = mn1;
        l_run[0] = l_run[0] * corr0 + (p0 + p1);
        l_run[1] = l_run[1] * corr1 + (p2 + p3);
        *reinterpret_cast<uint32_t*>(&sm.p16[pb][g * kPStride + e0]) = pack_half2(p0, p1);
        *reinterpret_cast<uint32_t*>(&sm.p16[pb][(g + 8) * kPStride + e0]) = pack_half2(p2, p3);
        *reinterpret_cast<uint32_t*>(&sm.pbf[pb][g * kPStride + e0]) = pack_bf162(p0, p1);
        *reinterpret_cast<uint32_t*>(&sm.pbf[pb][(g + 8) * kPStride + e0]) = pack_bf162(p2, p3);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            o[j][0] *= corr0;
            o[j][1] *= corr0;
            o[j][2] *= corr1;
            o[j][3] *= corr1;
        }
        __syncthreads();   // (B) P published

        // -- PV: this warp's 64 output dims; n-tile j, column g <-> dim base + 8g + j --
        const uint16_t* P = rope_warp ? sm.pbf[pb] : sm.p16[pb];
#pragma unroll
        for (int t = 0; t < kAT / 16; ++t) {
            uint32_t a0, a1, a2, a3;
            ldmatrix_x4(a0, a1, a2, a3, P + (lane & 15) * kPStride + 16 * t + ((lane >> 4) << 3));
            const int ea = 16 * t + 2 * cq;   // entries ea, ea+1 (b0) and ea+8, ea+9 (b1)
            if (!rope_warp) {
                const int off = 64 * warp + 8 * g;
                const uint2 A = *reinterpret_cast<const uint2*>(stg + (ea)*kEStride + off);
                const uint2 Bv = *reinterpret_cast<const uint2*>(stg + (ea + 1) * kEStride + off);
                const uint2 C = *reinterpret_cast<const uint2*>(stg + (ea + 8) * kEStride + off);
                const uint2 D = *reinterpret_cast<const uint2*>(stg + (ea + 9) * kEStride + off);
#pragma unroll
                for (int hw = 0; hw < 2; ++hw) {   // n-tiles 4hw .. 4hw+3
                    const uint32_t xa = hw ? A.y : A.x, xb = hw ? Bv.y : Bv.x;
                    const uint32_t xc = hw ? C.y : C.x, xd = hw ? D.y : D.x;
                    uint32_t bb0[4], bb1[4];
                    e4m3x4_to_f16x2x2(prmt(xa, xb, 0x5140u), bb0[0], bb0[1]);
                    e4m3x4_to_f16x2x2(prmt(xa, xb, 0x7362u), bb0[2], bb0[3]);
                    e4m3x4_to_f16x2x2(prmt(xc, xd, 0x5140u), bb1[0], bb1[1]);
                    e4m3x4_to_f16x2x2(prmt(xc, xd, 0x7362u), bb1[2], bb1[3]);
#pragma unroll
                    for (int j = 0; j < 4; ++j) mma_f16(o[4 * hw + j], a0, a1, a2, a3, bb0[j], bb1[j]);
                }
            } else {
                const int off = kNope + 16 * g;   // bf16 elements 8g..8g+7 of the RoPE part
                const uint4 A = *reinterpret_cast<const uint4*>(stg + (ea)*kEStride + off);
                const uint4 Bv = *reinterpret_cast<const uint4*>(stg + (ea + 1) * kEStride + off);
                const uint4 C = *reinterpret_cast<const uint4*>(stg + (ea + 8) * kEStride + off);
                const uint4 D = *reinterpret_cast<const uint4*>(stg + (ea + 9) * kEStride + off);
                const uint32_t wa[4] = {A.x, A.y, A.z, A.w}, wb[4] = {Bv.x, Bv.y, Bv.z, Bv.w};
                const uint32_t wc[4] = {C.x, C.y, C.z, C.w}, wd[4] = {D.x, D.y, D.z, D.w};
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const uint32_t sel = (j & 1) ? 0x7632u : 0x5410u;
                    mma_bf16(o[j], a0, a1, a2, a3, prmt(wa[j >> 1], wb[j >> 1], sel),
                             prmt(wc[j >> 1], wd[j >> 1], sel));
                }
            }
        }
        consumed = it + 1;
    }
    if (!ok) {
        // drain (bounded) the tiles produced beyond what was consumed, then stop
        for (int t = consumed; t < produced; ++t) (void)mbar_wait(&sm.full[t % kAStages], (t / kAStages) & 1);
        if (tid < kHeads) mlpart[part * kHeads + tid] = make_float2(-INFINITY, 0.f);
        return;
    }

    // ---- row sums across the 4 lanes of a group and the warps ---------------------
    float ls0 = l_run[0], ls1 = l_run[1];
    ls0 += __shfl_xor_sync(0xffffffffu, ls0, 1);
    ls0 += __shfl_xor_sync(0xffffffffu, ls0, 2);
    ls1 += __shfl_xor_sync(0xffffffffu, ls1, 1);
    ls1 += __shfl_xor_sync(0xffffffffu, ls1, 2);
    if (cq == 0) {
        sm.lsum[warp][g] = ls0;
        sm.lsum[warp][g + 8] = ls1;
    }
    __syncthreads();
    if (warp == 0 && cq == 0) {
        float t0 = 0.f, t1 = 0.f;
        for (int w = 0; w < kWarps; ++w) {
            t0 += sm.lsum[w][g];
            t1 += sm.lsum[w][g + 8];
        }
        mlpart[part * kHeads + g] = make_float2(m_run[0], t0);
        mlpart[part * kHeads + g + 8] = make_float2(m_run[1], t1);
    }
    // ---- unnormalised O of this split ------------------------------------------------------
    float* ob = opart + part * kHeads * kDim;
    const int base = 64 * warp;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int d0 = base + 8 * (2 * cq) + j, d1 = base + 8 * (2 * cq + 1) + j;
        ob[g * kDim + d0] = o[j][0];
        ob[g * kDim + d1] = o[j][1];
        ob[(g + 8) * kDim + d0] = o[j][2];
        ob[(g + 8) * kDim + d1] = o[j][3];
    }
}

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
    const int64_t tiles = (L + kAT - 1) / kAT;
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
    const size_t smem = sizeof(AttnSmem);
    cudaError_t e = set_smem_once(attention_partial_kernel, smem);
    if (e != cudaSuccess) return e;
    dim3 grid(plan.splits, B);
    attention_partial_kernel<<<grid, kAttnThreads, smem, stream>>>(q, comp_kv, cap, ratio, topk, k,
                                                                   win_kv, W, seq_len, scale,
                                                                   plan.splits, opart, mlpart, err);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    attention_merge_kernel<<<dim3(B, kHeads), 128, 0, stream>>>(opart, mlpart, plan.splits, out, lse_out);
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
