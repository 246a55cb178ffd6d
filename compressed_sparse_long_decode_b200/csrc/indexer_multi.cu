// Multi-query lightning indexer: Q query tokens of one sequence (a speculative or multi-token
// prediction draft, or a prefill chunk) scored against the FP4 key cache in ONE pass over the
// keys, then an exact top-k per query.
//
// Source: "DeepSeek-V4: a million-token context that agents can actually use" -- CSA paragraph
// (FP4, ReLU-scored multi-head dot product of each query against the 4x-compressed entries; the
// top-k compressed blocks per query), layer-pattern paragraph (the multi-token-prediction block
// runs several query tokens per step).  Query j of sequence b stands at raw position
// p = seq_len[b] - Q + j and sees the entries s < min((p + 1) / ratio, cap) (an entry is visible
// once its last token is in).  Every query's score and selection are those indexer_topk forms
// for it alone (same FP4 quantisation, exact integer group dots, same fp32 operation order, ties
// to the lower index), so the result equals Q separate indexer_topk calls.
//
// 1. indexer_multi_score_kernel -- persistent CTAs over 128-entry tiles of every sequence.  A
//    copy warp streams the key codes and scales with 1-D bulk copies, eight tiles (32 KB + 8 KB)
//    per copy, three copies in flight; one thread issues one tcgen05.mma kind::mxf4 per tile
//    (M = 128 entries, N = 8 Q rows of the query operand: row 8q + 4g + h holds group g of head
//    h of query q, the other group zero, so each output column is one exact group dot) into one
//    of six accumulator slots; three warpgroups take the tiles in turn, read the dots back
//    (thread = entry), form every query's fp32 score and write its order key to the workspace,
//    and add the keys' top 11 bits to per-query histograms, which the CTA adds into global ones
//    at the end.
// 2. indexer_multi_gather_kernel -- P CTAs per (sequence, query), each over one contiguous part
//    of the query's keys: the threshold bin from the global histogram, then the keys of that bin
//    and above, with their indices, compacted in index order into the part's candidate list.
// 3. indexer_multi_select_kernel -- one CTA per (sequence, query): the P lists, concatenated in
//    part order (so still in index order), go to shared memory; two more radix levels
//    (11 + 10 bits) there, then the entries in index order: every key above the threshold and
//    the first ones equal to it.  It zeroes the histogram it used, so the workspace stays ready
//    for the next call.
#include "csld_internal.cuh"
#include "kernels.cuh"
#include "sm100.cuh"

namespace csld {

namespace {

constexpr int kMqThreads = 512;          // warps 0-11 epilogue (3 warpgroups), warp 12 copies, warp 13 MMA
constexpr int kMqTile = 128;             // entries per MMA (M)
constexpr int kMqGroupTiles = 8;         // tiles per bulk copy
constexpr int kMqGroup = kMqTile * kMqGroupTiles;   // 1024 entries per copy group
constexpr int kMqStages = 3;             // copy groups in flight
constexpr int kMqBins = 2048;            // histogram of the keys' top 11 bits
constexpr int kMqEpi = 3;                // epilogue warpgroups: tile t goes to warpgroup t % 3
constexpr int kMqSlots = 6;              // accumulator slots (tile t uses slot t % 6), 64 columns each
constexpr uint32_t kMqTmemCols = 512;    // 6 x 64 columns (8 Q <= 64), scale factors at 384
constexpr uint32_t kMqSfCol = 384;
constexpr int kMqCopyWarp = 12, kMqMmaWarp = 13;

struct MqSmem {
    uint8_t codes[kMqStages][kMqGroup * kIkey];     // 32 KB per group, stored (pre-swizzled) layout
    float scales[kMqStages][kMqGroup * 2];          // 8 KB per group
    // query operand: 32-byte rows with the 32-byte swizzle (shared keys), or 128-byte rows with
    // the 128-byte swizzle (per-head keys: head h's codes in the row's 32-byte slice h)
    alignas(1024) uint8_t bq[8 * CSLD_MULTI_MAX_Q * kIkey * kIdxHeads];
    float qscale[CSLD_MULTI_MAX_Q][8];              // [q][group * 4 + head]
    float hw[CSLD_MULTI_MAX_Q][kIdxHeads];          // head weights of each query
    int64_t nq[CSLD_MULTI_MAX_Q];                   // entries query q sees
    uint32_t hist[CSLD_MULTI_MAX_Q][kMqBins];
    uint64_t full[kMqStages], gfree[kMqStages], accf[kMqSlots], sfree[kMqSlots], drain;
    uint32_t tmem_base;
    int32_t fail, n_mma;
};

}  // namespace

// Grid (chunks, B): CTA (c, b) scores tiles c, c + chunks, ... of sequence b's visible range.
// kKeyHeads = 1: one key shared by the 4 heads (32 code bytes + 2 scales per entry, 1,024-entry
// copy groups).  kKeyHeads = 4: per-head keys (128 code bytes in 128-byte-swizzle rows + 8
// scales per entry, 256-entry copy groups; one MMA per head and tile, each over the head's
// 32-byte K slice of the keys and of the query operand, whose other heads' rows are zero there,
// so the output columns are the same exact group dots).
template <int kKeyHeads>
__global__ void __launch_bounds__(kMqThreads, 1) indexer_multi_score_kernel(
    const uint8_t* __restrict__ ikeys, const float* __restrict__ iscales, int64_t cap,
    const int32_t* __restrict__ seq_len, int ratio, const float* __restrict__ q_idx,
    const float* __restrict__ head_w, int Q, uint32_t* __restrict__ keys_out, uint32_t* __restrict__ ghist,
    int32_t* err) {
    constexpr int kKeyBytes = kIkey * kKeyHeads;           // code bytes per entry
    constexpr int kSf = 2 * kKeyHeads;                     // scales per entry
    constexpr int kGroupE = kMqGroup / kKeyHeads;          // entries per copy group (32 KB of codes)
    constexpr int kGroupTiles = kGroupE / kMqTile;
    extern __shared__ __align__(128) uint8_t smem_raw[];
    MqSmem& sm = *reinterpret_cast<MqSmem*>(smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023));
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = blockIdx.y, chunks = gridDim.x, c = blockIdx.x;
    if (tid == 0) {
        for (int s = 0; s < kMqStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.gfree[s], 4 * kMqEpi);   // every epilogue warp, once per copy group
        }
        for (int s = 0; s < kMqSlots; ++s) {
            mbar_init(&sm.accf[s], 1);
            mbar_init(&sm.sfree[s], 4);            // the 4 warps of the slot's warpgroup
        }
        mbar_init(&sm.drain, 1);
        sm.fail = 0;
        sm.n_mma = 0;
        fence_barrier_init();
    }
    if (warp == kMqMmaWarp) {
        tmem_alloc(&sm.tmem_base, kMqTmemCols);
        tmem_relinquish();
    }
    for (int i = tid; i < Q * kMqBins; i += kMqThreads) (&sm.hist[0][0])[i] = 0u;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    pdl_wait();      // lengths, keys and queries come from upstream
    pdl_trigger();
    const uint32_t tmem = sm.tmem_base;
    volatile int32_t* fail = &sm.fail;

    int32_t n = seq_len[b];
    if (n < 0) {
        if (tid == 0 && c == 0) dev_error(err, CSLD_DEVERR_SEQ_LEN);
        n = 0;
    }
    // the newest query sees the most entries; query q sees n_q of them
    const int64_t n_max = min64(n / ratio, cap);
    if (tid < Q) {
        sm.nq[tid] = min64((int64_t)(n - Q + tid + 1) / ratio, cap);
#pragma unroll
        for (int h = 0; h < kIdxHeads; ++h) sm.hw[tid][h] = __ldg(head_w + ((size_t)b * Q + tid) * kIdxHeads + h);
    }
    __syncthreads();
    const int n_tiles_all = static_cast<int>((n_max + kMqTile - 1) / kMqTile);
    // this CTA's tiles: whole copy groups g = c, c + chunks, ...
    const int n_groups_all = (n_tiles_all + kGroupTiles - 1) / kGroupTiles;
    const int my_groups = n_groups_all > c ? (n_groups_all - c + chunks - 1) / chunks : 0;
    const uint8_t* cbase = ikeys + (size_t)b * cap * kKeyBytes;
    const float* sbase = iscales + (size_t)b * cap * kSf;

    // ---- query operand (warps 0-3, then handed to the MMA warp; the copy warp starts at once) --
    if (warp < 4 && kKeyHeads > 1) {
        // per-head keys: 8Q rows of 128 bytes, zero but for the 16 bytes of row n = 8q + 4g + h
        // that hold group g of head h of query q, at byte 32h + 16g of the row (16-byte chunk
        // 2h + g, stored at chunk (2h + g) ^ (n mod 8))
        for (int i = tid; i < 8 * Q * kIkey * kIdxHeads / 4; i += 128) reinterpret_cast<uint32_t*>(sm.bq)[i] = 0u;
        named_barrier(2, 128);
        for (int t = tid; t < 32 * Q; t += 128) {   // thread (n, jj): bytes 4jj .. 4jj+3 of the 16
            const int n_row = t >> 2, jj = t & 3;
            const int q = n_row >> 3, r8 = n_row & 7, h = r8 & 3, grp = r8 >> 2;
            const float* qv = q_idx + (((size_t)b * Q + q) * kIdxHeads + h) * kIdxDim + 32 * grp;
            float amax = 0.f;
            for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(__ldg(qv + i)));
            const float sg = fp4_group_scale(amax);
            const float inv = 1.0f / sg;   // exact: a power of two
            uint32_t word = 0u;
#pragma unroll
            for (int i = 0; i < 8; ++i) word |= e2m1_code(__ldg(qv + 8 * jj + i) * inv) << (4 * i);
            *reinterpret_cast<uint32_t*>(sm.bq + n_row * (kIkey * kIdxHeads) + 16 * ((2 * h + grp) ^ r8) + 4 * jj) = word;
            if (jj == 0) sm.qscale[q][grp * 4 + h] = sg;
        }
        fence_proxy_async_smem();
        tmem_st_32x32b_x8_fill(tmem + ((32u * warp) << 16) + kMqSfCol, 0x7F7F7F7Fu);
        tmem_st_32x32b_x8_fill(tmem + ((32u * warp) << 16) + kMqSfCol + 8, 0x7F7F7F7Fu);
        tmem_st_wait();
    } else if (warp < 4) {
        // thread t < 8 Q writes row n = t / 8 ... one row per 8 threads: thread (n, j) writes
        // bytes 4j .. 4j+3 of row n
        for (int t = tid; t < 64 * Q; t += 128) {
            const int n_row = t >> 3, j = t & 7;
            const int q = n_row >> 3, r8 = n_row & 7, h = r8 & 3, grp = r8 >> 2;
            const float* qv = q_idx + (((size_t)b * Q + q) * kIdxHeads + h) * kIdxDim + 32 * grp;
            float amax = 0.f;
            for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(__ldg(qv + i)));
            const float sg = fp4_group_scale(amax);
            const float inv = 1.0f / sg;   // exact: a power of two
            uint32_t word = 0u;
            if ((j >> 2) == grp) {   // bytes 4j..4j+3 hold elements 8(j&3) .. 8(j&3)+7 of group grp
#pragma unroll
                for (int i = 0; i < 8; ++i) word |= e2m1_code(__ldg(qv + 8 * (j & 3) + i) * inv) << (4 * i);
            }
            const int half = (j >> 2) ^ ((n_row >> 2) & 1);
            *reinterpret_cast<uint32_t*>(sm.bq + n_row * kIkey + half * 16 + (j & 3) * 4) = word;
            if (j == 0) sm.qscale[q][grp * 4 + h] = sg;
        }
        fence_proxy_async_smem();
        // unit block-scale factors (UE8M0 0x7F = 2^0) for A and B, every lane
        tmem_st_32x32b_x8_fill(tmem + ((32u * warp) << 16) + kMqSfCol, 0x7F7F7F7Fu);
        tmem_st_32x32b_x8_fill(tmem + ((32u * warp) << 16) + kMqSfCol + 8, 0x7F7F7F7Fu);
        tmem_st_wait();
    }
    if (warp < 4 || warp == kMqMmaWarp) {   // query operand and scale factors ready (warps 0-3 and the MMA warp)
        tc_fence_before();
        named_barrier(1, 5 * 32);
        tc_fence_after();
    }

    if (warp == kMqCopyWarp) {
        if (lane == 0) {
            for (int i = 0; i < my_groups; ++i) {
                const int s = i % kMqStages;
                if (*fail) break;
                if (i >= kMqStages && !mbar_wait(&sm.gfree[s], ((i / kMqStages) - 1) & 1)) {
                    *fail = 1;
                    break;
                }
                const int64_t e0 = (int64_t)(c + i * chunks) * kGroupE;
                const int ne = static_cast<int>(min64(kGroupE, n_max - e0));
                const uint32_t cb = static_cast<uint32_t>(ne) * kKeyBytes;
                // scales: 8 bytes per entry (an even count: cap is even) or 32 per entry
                const uint32_t sb = kKeyHeads == 1 ? static_cast<uint32_t>((ne + 1) & ~1) * 8u
                                                   : static_cast<uint32_t>(ne) * 4u * kSf;
                mbar_arrive_expect_tx(&sm.full[s], cb + sb);
                bulk_g2s(sm.codes[s], cbase + (size_t)e0 * kKeyBytes, cb, &sm.full[s]);
                bulk_g2s(sm.scales[s], sbase + (size_t)e0 * kSf, sb, &sm.full[s]);
            }
        }
    } else if (warp == kMqMmaWarp) {
        if (lane == 0) {
            const uint64_t bdesc = smem_desc_kmajor_sw32(sm.bq);
            const uint32_t idesc = idesc_mxf4_m128(static_cast<uint32_t>(8 * Q));
            int t = 0;
            for (int i = 0; i < my_groups && !*fail; ++i) {
                const int s = i % kMqStages;
                if (!mbar_wait(&sm.full[s], (i / kMqStages) & 1)) {
                    *fail = 1;
                    break;
                }
                tc_fence_after();
                const int g = c + i * chunks;
                const int nt = min(kGroupTiles, n_tiles_all - g * kGroupTiles);
                for (int tt = 0; tt < nt; ++tt, ++t) {
                    const int slot = t % kMqSlots;
                    if (t >= kMqSlots && !mbar_wait(&sm.sfree[slot], ((t / kMqSlots) - 1) & 1)) {
                        *fail = 1;
                        break;
                    }
                    tc_fence_after();
                    if constexpr (kKeyHeads == 1) {
                        umma_mxf4(tmem + 64u * slot, smem_desc_kmajor_sw32(sm.codes[s] + tt * kMqTile * kIkey), bdesc,
                                  idesc, tmem + kMqSfCol, tmem + kMqSfCol + 8, 0u);
                    } else {
                        const uint64_t ad = desc_sw128(sm.codes[s] + tt * kMqTile * kKeyBytes, 0);
                        const uint64_t bd = desc_sw128(sm.bq, 0);
#pragma unroll
                        for (int h = 0; h < kKeyHeads; ++h)   // head h: the 32-byte K slice h
                            umma_mxf4(tmem + 64u * slot, ad + (32 * h) / 16, bd + (32 * h) / 16, idesc, tmem + kMqSfCol,
                                      tmem + kMqSfCol + 8, h > 0 ? 1u : 0u);
                    }
                    umma_commit(&sm.accf[slot]);
                }
                if (*fail) break;
            }
            sm.n_mma = t;
        }
    } else if (warp < 4 * kMqEpi) {
        // ---- epilogue: warpgroup wg takes tiles wg, wg + 3, ...; thread = entry m of the tile ---
        const int wg = warp >> 2, quad = warp & 3;
        const int m = 32 * quad + lane;
        const uint32_t lane_addr = tmem + ((32u * quad) << 16);
        int t = 0;
        for (int i = 0; i < my_groups; ++i) {
            const int s = i % kMqStages;
            const int g = c + i * chunks;
            const int nt = min(kGroupTiles, n_tiles_all - g * kGroupTiles);
            bool ok = true;
            for (int tt = 0; tt < nt; ++tt, ++t) {
                if (t % kMqEpi != wg) continue;
                const int slot = t % kMqSlots;
                ok = !*fail && mbar_wait(&sm.accf[slot], (t / kMqSlots) & 1);
                if (!__all_sync(0xffffffffu, ok)) {
                    if (lane == 0) *fail = 1;
                    ok = false;
                    break;
                }
                tc_fence_after();
                const int64_t e = (int64_t)g * kGroupE + tt * kMqTile + m;
                // key scales of this entry: (group 0, group 1) of the shared key or of each head's
                const float* ksp = sm.scales[s] + (size_t)(tt * kMqTile + m) * kSf;
                for (int q0 = 0; q0 < Q; q0 += 2) {   // two queries (16 columns) per load
                    uint32_t r[16];
                    tmem_ld_32x32b_x16(lane_addr + 64u * slot + 8u * q0, r);
                    tmem_ld_wait();
#pragma unroll
                    for (int qq = 0; qq < 2; ++qq) {
                        const int q = q0 + qq;
                        if (q >= Q) break;
                        const int64_t n_q = sm.nq[q];
                        float rr[4];
#pragma unroll
                        for (int h = 0; h < 4; ++h) {
                            // d = fma(I1, s1, I0*s0) with s_g = (qscale_g * kscale_g) * 0.25
                            const float i0 = __fmul_rn(__uint_as_float(r[8 * qq + h]), 4.0f);
                            const float i1 = __fmul_rn(__uint_as_float(r[8 * qq + 4 + h]), 4.0f);
                            const int kh = kKeyHeads == 1 ? 0 : 2 * h;
                            const float s0 = __fmul_rn(__fmul_rn(sm.qscale[q][h], ksp[kh]), 0.25f);
                            const float s1 = __fmul_rn(__fmul_rn(sm.qscale[q][4 + h], ksp[kh + 1]), 0.25f);
                            const float d = __fmaf_rn(i1, s1, __fmul_rn(i0, s0));
                            rr[h] = d > 0.f ? d : 0.f;
                        }
                        const float* w = sm.hw[q];
                        float sc = __fmul_rn(w[0], rr[0]);
                        sc = __fmaf_rn(w[1], rr[1], sc);
                        sc = __fmaf_rn(w[2], rr[2], sc);
                        sc = __fmaf_rn(w[3], rr[3], sc);
                        const uint32_t key = score_key(sc);
                        if (e < n_q) {
                            keys_out[((size_t)b * Q + q) * cap + (size_t)e] = key;
                            atomicAdd(&sm.hist[q][key >> 21], 1u);
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.sfree[slot]);
            }
            if (!ok) break;
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.gfree[s]);   // the group's codes and scales are consumed
        }
    }
    tc_fence_before();
    __syncthreads();
    if (sm.fail) {
        // a bounded wait gave up: record it and let the MMAs in flight finish before the tensor
        // memory is released (the histograms of this call are then incomplete; zero the
        // workspace again, as for indexer_topk)
        if (warp == kMqMmaWarp && lane == 0) {
            dev_error(err, CSLD_DEVERR_TIMEOUT);
            umma_commit(&sm.drain);
            (void)mbar_wait(&sm.drain, 0);
        }
        __syncthreads();
    }
    // this CTA's histograms into the global ones
    for (int i = tid; i < Q * kMqBins; i += kMqThreads) {
        const uint32_t v = (&sm.hist[0][0])[i];
        if (v) atomicAdd(ghist + (size_t)b * Q * kMqBins + i, v);
    }
    if (warp == kMqMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kMqTmemCols);
    }
}

namespace {


// Block-wide exclusive scan of v (1024 threads); *total = the sum.
__device__ __forceinline__ uint32_t mq_block_scan(uint32_t v, uint32_t* red, uint32_t* total) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint32_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) red[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const uint32_t w = red[lane];
        uint32_t wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += y;
        }
        red[32 + lane] = wi - w;
        if (lane == 31) red[64] = wi;
    }
    __syncthreads();
    const uint32_t r = red[32 + warp] + incl - v;
    *total = red[64];
    __syncthreads();
    return r;
}

// The bin of nb bins (counts in smem h) holding the want-th largest key and how many keys are
// wanted inside it, in sel[0..1] (bin 0 and want when the counts fall short: an incomplete
// histogram).  The whole block (1024 threads; nb a multiple of it, at most 2 bins per thread):
// thread t holds the bins at places per t .. per t + per - 1 from the top, and a block scan of
// their counts finds the thread whose bins hold the want-th key.  Ends with a barrier.
__device__ void mq_find_bin_block(const uint32_t* h, int nb, uint32_t want, uint32_t* red, uint32_t* sel) {
    const int tid = threadIdx.x;
    const int per = nb / static_cast<int>(blockDim.x);
    uint32_t c[2] = {0u, 0u}, tot = 0u;
    for (int j = 0; j < per; ++j) {
        c[j] = h[nb - 1 - (per * tid + j)];
        tot += c[j];
    }
    if (tid == 0) {   // defaults if the counts fall short (an incomplete histogram)
        sel[0] = 0u;
        sel[1] = want;
    }
    uint32_t total;
    const uint32_t excl = mq_block_scan(tot, red, &total);
    if (excl < want && excl + tot >= want) {
        uint32_t run = excl;
        for (int j = 0; j < per; ++j) {
            if (run + c[j] >= want) {
                sel[0] = static_cast<uint32_t>(nb - 1 - (per * tid + j));
                sel[1] = want - run;
                break;
            }
            run += c[j];
        }
    }
    __syncthreads();
}

}  // namespace

// Grid (Q, B), 1024 threads: the exact top-k of query q of sequence b.  The keys of the
// threshold bin (found from the scoring histogram) and above are gathered into shared memory
// in index order by one pass over the query's keys (sixteen per thread at a time, 16-byte
// loads); the last two radix levels and the emission then run in shared memory.  When they do
// not fit (more than kMqCand keys: heavy ties), the levels and the emission read the keys from
// global memory instead.
constexpr int kMqSelThreads = 1024;
constexpr int kMqPer = 16;                       // keys per thread per pass step
constexpr int kMqCand = 20480;                   // candidates kept in shared memory
struct MqSelSmem {
    uint32_t ckey[kMqCand];
    uint32_t cidx[kMqCand];
    uint32_t h[kMqBins];
    uint32_t sel[4];
    uint32_t red[96];
};

// Grid (P, Q, B), 1024 threads: part p of query q of sequence b.  The query's keys are walked in
// steps of kMqSelThreads * kMqPer; part p takes steps [S p / P, S (p + 1) / P).  Keys of the
// threshold bin and above go to the part's list as (key, index) in index order; the count goes
// to counts.  When the candidates of the whole query would not fit in the select kernel's shared
// memory (heavy ties) nothing is gathered: the select kernel then reads the keys itself.
struct MqGatherSmem {
    uint32_t h[kMqBins];
    uint32_t sel[4];
    uint32_t red[96];
};
__global__ void __launch_bounds__(kMqSelThreads) indexer_multi_gather_kernel(const uint32_t* __restrict__ keys,
                                                                             int64_t cap,
                                                                             const int32_t* __restrict__ seq_len,
                                                                             int ratio, int Q, int k, int P,
                                                                             const uint32_t* __restrict__ ghist,
                                                                             uint2* __restrict__ lists,
                                                                             uint32_t* __restrict__ counts) {
    __shared__ MqGatherSmem sm;
    const int p = blockIdx.x, q = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
    pdl_wait();
    pdl_trigger();
    int32_t n = seq_len[b];
    if (n < 0) n = 0;
    const int64_t pos1 = (int64_t)n - Q + q + 1;
    const int64_t n_q = pos1 > 0 ? min64(pos1 / ratio, cap) : 0;
    const size_t row = (size_t)b * Q + q;
    if (n_q <= k) return;   // the select kernel lists every visible entry
    const uint32_t* gh = ghist + row * kMqBins;
    for (int i = tid; i < kMqBins; i += blockDim.x) sm.h[i] = __ldcg(gh + i);
    __syncthreads();
    mq_find_bin_block(sm.h, kMqBins, static_cast<uint32_t>(k), sm.red, sm.sel);
    const uint32_t b1 = sm.sel[0], need1 = sm.sel[1];
    if (static_cast<uint32_t>(k) - need1 + sm.h[b1] > static_cast<uint32_t>(kMqCand)) return;
    const uint32_t lo1 = b1 << 21;
    const uint32_t* kq = keys + row * cap;
    const int64_t pcap = min64(kMqCand, cap);   // a part's list holds at most this many
    uint2* list = lists + (row * P + p) * pcap;
    constexpr int64_t kStep = (int64_t)kMqSelThreads * kMqPer;
    const int64_t steps = (n_q + kStep - 1) / kStep;
    const int64_t i_lo = steps * p / P * kStep, i_hi = min64(steps * (p + 1) / P * kStep, n_q);
    const bool vec = ((reinterpret_cast<uintptr_t>(kq) & 15u) == 0);
    uint32_t n_c = 0u;
    for (int64_t base = i_lo; base < i_hi; base += kStep) {
        const int64_t i0 = base + (int64_t)tid * kMqPer;
        uint32_t v[kMqPer];
        if (vec && i0 + kMqPer <= i_hi) {
#pragma unroll
            for (int j = 0; j < kMqPer / 4; ++j) {
                const uint4 x = __ldcg(reinterpret_cast<const uint4*>(kq + i0) + j);
                v[4 * j] = x.x;
                v[4 * j + 1] = x.y;
                v[4 * j + 2] = x.z;
                v[4 * j + 3] = x.w;
            }
        } else {
#pragma unroll
            for (int j = 0; j < kMqPer; ++j) v[j] = i0 + j < i_hi ? __ldcg(kq + i0 + j) : 0u;
        }
        uint32_t cnt = 0u;
#pragma unroll
        for (int j = 0; j < kMqPer; ++j) cnt += (i0 + j < i_hi && v[j] >= lo1) ? 1u : 0u;
        uint32_t tot;
        uint32_t at = n_c + mq_block_scan(cnt, sm.red, &tot);
#pragma unroll
        for (int j = 0; j < kMqPer; ++j)
            if (i0 + j < i_hi && v[j] >= lo1) {
                if (at < static_cast<uint32_t>(pcap)) list[at] = make_uint2(v[j], static_cast<uint32_t>(i0 + j));
                ++at;
            }
        n_c += tot;
    }
    if (tid == 0) counts[row * P + p] = min(n_c, static_cast<uint32_t>(pcap));
}

__global__ void __launch_bounds__(kMqSelThreads) indexer_multi_select_kernel(const uint32_t* __restrict__ keys,
                                                                             int64_t cap,
                                                                             const int32_t* __restrict__ seq_len,
                                                                             int ratio, int Q, int k, int P,
                                                                             uint32_t* __restrict__ ghist,
                                                                             const uint2* __restrict__ lists,
                                                                             const uint32_t* __restrict__ counts,
                                                                             int32_t* __restrict__ topk_out) {
    extern __shared__ __align__(16) uint8_t sel_raw[];
    MqSelSmem& sm = *reinterpret_cast<MqSelSmem*>(sel_raw);
    uint32_t* h = sm.h;
    uint32_t* sel = sm.sel;
    uint32_t* red = sm.red;
    const int q = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
    pdl_wait();
    pdl_trigger();
    int32_t n = seq_len[b];
    if (n < 0) n = 0;
    const int64_t pos1 = (int64_t)n - Q + q + 1;                      // tokens this query sees
    const int64_t n_q = pos1 > 0 ? min64(pos1 / ratio, cap) : 0;
    const uint32_t* kq = keys + ((size_t)b * Q + q) * cap;
    uint32_t* gh = ghist + ((size_t)b * Q + q) * kMqBins;
    int32_t* out = topk_out + ((size_t)b * Q + q) * k;
    for (int i = tid; i < kMqBins; i += blockDim.x) {
        h[i] = gh[i];
        gh[i] = 0u;    // ready for the next call
    }
    __syncthreads();
    if (n_q <= k) {
        for (int64_t i = tid; i < k; i += blockDim.x) out[i] = i < n_q ? static_cast<int32_t>(i) : -1;
        return;
    }
    // level 1 (bits 31..21) from the scoring histogram
    mq_find_bin_block(h, kMqBins, static_cast<uint32_t>(k), red, sel);
    const uint32_t b1 = sel[0], need1 = sel[1];
    const uint32_t above1 = static_cast<uint32_t>(k) - need1;   // keys above bin b1
    const uint32_t in1 = h[b1];                                  // keys in it
    __syncthreads();
    const bool in_smem = above1 + in1 <= static_cast<uint32_t>(kMqCand);
    // ---- the keys of bin >= b1 in index order (when they fit): the parts' lists, in order ------
    uint32_t n_c = 0u;
    if (in_smem) {
        const size_t row = (size_t)b * Q + q;
        if (tid < P) red[32 + tid] = __ldcg(counts + row * P + tid);
        __syncthreads();
        if (tid == 0) {   // red[pp] = where part pp's keys start; red[P] = all
            uint32_t acc = 0u;
            for (int pp = 0; pp < P; ++pp) {
                red[pp] = acc;
                acc += red[32 + pp];
            }
            red[P] = acc;
        }
        __syncthreads();
        n_c = min(red[P], static_cast<uint32_t>(kMqCand));   // equal whenever the histogram is exact
        for (uint32_t j0 = 0; j0 < n_c; j0 += 4u * kMqSelThreads) {
            uint2 e[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const uint32_t j = j0 + u * kMqSelThreads + tid;
                e[u] = make_uint2(0u, 0u);
                if (j < n_c) {
                    int pp = 0;
                    while (pp + 1 < P && red[pp + 1] <= j) ++pp;
                    e[u] = __ldcg(lists + (row * P + pp) * min64(kMqCand, cap) + (j - red[pp]));
                }
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const uint32_t j = j0 + u * kMqSelThreads + tid;
                if (j < n_c) {
                    sm.ckey[j] = e[u].x;
                    sm.cidx[j] = e[u].y;
                }
            }
        }
        __syncthreads();
    }
    // ---- levels 2 (bits 20..10) and 3 (bits 9..0) inside bin b1 --------------------------------
    for (int i = tid; i < kMqBins; i += blockDim.x) h[i] = 0u;
    __syncthreads();
    if (in_smem) {
        for (uint32_t i = tid; i < n_c; i += blockDim.x)
            if ((sm.ckey[i] >> 21) == b1) atomicAdd(&h[(sm.ckey[i] >> 10) & 2047u], 1u);
    } else {
        for (int64_t i = tid; i < n_q; i += blockDim.x) {
            const uint32_t key = __ldcg(kq + i);
            if ((key >> 21) == b1) atomicAdd(&h[(key >> 10) & 2047u], 1u);
        }
    }
    __syncthreads();
    mq_find_bin_block(h, kMqBins, need1, red, sel);
    const uint32_t b2 = sel[0], need2 = sel[1];
    __syncthreads();
    for (int i = tid; i < 1024; i += blockDim.x) h[i] = 0u;
    __syncthreads();
    const uint32_t top22 = (b1 << 11) | b2;
    if (in_smem) {
        for (uint32_t i = tid; i < n_c; i += blockDim.x)
            if ((sm.ckey[i] >> 10) == top22) atomicAdd(&h[sm.ckey[i] & 1023u], 1u);
    } else {
        for (int64_t i = tid; i < n_q; i += blockDim.x) {
            const uint32_t key = __ldcg(kq + i);
            if ((key >> 10) == top22) atomicAdd(&h[key & 1023u], 1u);
        }
    }
    __syncthreads();
    mq_find_bin_block(h, 1024, need2, red, sel);
    const uint32_t thr = (top22 << 10) | sel[0], take_eq = sel[1];
    __syncthreads();
    // ---- emit in index order: keys above the threshold, and the first take_eq equal to it -----
    if (in_smem) {
        // thread t takes candidates [per t, per (t + 1)); one block scan of its (above, equal)
        // counts, packed into one word (each below 2^16), gives where its entries go
        const uint32_t per = (n_c + kMqSelThreads - 1) / kMqSelThreads;
        const uint32_t c0 = min(n_c, per * static_cast<uint32_t>(tid)), c1 = min(n_c, c0 + per);
        uint32_t gt = 0u, eq = 0u;
        for (uint32_t i = c0; i < c1; ++i) {
            gt += sm.ckey[i] > thr ? 1u : 0u;
            eq += sm.ckey[i] == thr ? 1u : 0u;
        }
        uint32_t tot;
        const uint32_t pre = mq_block_scan((gt << 16) | eq, red, &tot);
        uint32_t at = (pre >> 16) + min(pre & 0xFFFFu, take_eq), e_seen = pre & 0xFFFFu;
        for (uint32_t i = c0; i < c1; ++i) {
            const uint32_t key = sm.ckey[i];
            bool take = key > thr;
            if (key == thr) take = e_seen++ < take_eq;
            if (take) {
                if (at < static_cast<uint32_t>(k)) out[at] = static_cast<int32_t>(sm.cidx[i]);
                ++at;
            }
        }
        return;
    }
    const int64_t n_e = n_q;
    uint32_t base_sel = 0u, base_eq = 0u;
    for (int64_t i0 = 0; i0 < n_e; i0 += blockDim.x) {
        const int64_t i = i0 + tid;
        uint32_t key = 0u, idx = 0u;
        if (i < n_e) {
            key = __ldcg(kq + i);
            idx = static_cast<uint32_t>(i);
        }
        const uint32_t eq = (i < n_e && key == thr) ? 1u : 0u;
        uint32_t eq_tot;
        const uint32_t eq_before = base_eq + mq_block_scan(eq, red, &eq_tot);
        const uint32_t take = (i < n_e && key > thr) || (eq && eq_before < take_eq) ? 1u : 0u;
        uint32_t take_tot;
        const uint32_t at = base_sel + mq_block_scan(take, red, &take_tot);
        if (take && at < static_cast<uint32_t>(k)) out[at] = static_cast<int32_t>(idx);
        base_sel += take_tot;
        base_eq += eq_tot;
        if (base_sel >= static_cast<uint32_t>(k)) break;   // uniform: every thread sees the same totals
    }
}

size_t indexer_multi_smem_bytes() { return sizeof(MqSmem) + 1024; }

// Parts per (sequence, query) of the gather: about one CTA per SM in all, at most 16.
int indexer_multi_parts(int B, int Q, int num_sms) {
    const int rows = max(B * Q, 1);
    return max(1, min(16, num_sms / rows));
}

// Workspace: the order keys [B][Q][cap], the histograms [B][Q][2048], the parts' candidate
// counts [B][Q][P] and lists [B][Q][P][min(kMqCand, cap)] of (key, index).
size_t indexer_multi_ws_bytes(int B, int Q, int64_t cap, int num_sms) {
    const size_t rows = (size_t)B * Q, P = (size_t)indexer_multi_parts(B, Q, num_sms);
    auto up = [](size_t x) { return (x + 255) / 256 * 256; };
    return up(rows * (size_t)cap * 4) + up(rows * kMqBins * 4) + up(rows * P * 4) +
           rows * P * (size_t)min64(kMqCand, cap) * sizeof(uint2);
}

cudaError_t launch_indexer_multi(const uint8_t* ikeys, const float* iscales, int64_t cap, const int32_t* seq_len,
                                 int ratio, const float* q_idx, const float* head_w, int B, int Q, int k,
                                 int32_t* topk_out, void* ws, int num_sms, int32_t* err, cudaStream_t stream,
                                 bool perhead) {
    const int P = indexer_multi_parts(B, Q, num_sms);
    const size_t rows = (size_t)B * Q;
    auto up = [](size_t x) { return (x + 255) / 256 * 256; };
    uint8_t* w8 = static_cast<uint8_t*>(ws);
    uint32_t* keys = reinterpret_cast<uint32_t*>(w8);
    uint32_t* ghist = reinterpret_cast<uint32_t*>(w8 + up(rows * (size_t)cap * 4));
    uint32_t* counts = reinterpret_cast<uint32_t*>(w8 + up(rows * (size_t)cap * 4) + up(rows * kMqBins * 4));
    uint2* lists = reinterpret_cast<uint2*>(w8 + up(rows * (size_t)cap * 4) + up(rows * kMqBins * 4) + up(rows * P * 4));
    const size_t smem = indexer_multi_smem_bytes();
    auto score = perhead ? indexer_multi_score_kernel<kIdxHeads> : indexer_multi_score_kernel<1>;
    cudaError_t e = set_smem_once(score, smem);
    if (e != cudaSuccess) return e;
    // copy groups of every sequence spread over about one CTA per SM
    const int64_t group_e = perhead ? kMqGroup / kIdxHeads : kMqGroup;
    const int64_t groups = (cap + group_e - 1) / group_e;
    int64_t chunks = max64(1, num_sms / max(B, 1));
    chunks = min64(chunks, groups);
    e = launch_pdl(score, dim3(static_cast<unsigned>(chunks), B), dim3(kMqThreads), smem, stream,
                   ikeys, iscales, cap, seq_len, ratio, q_idx, head_w, Q, keys, ghist, err);
    if (e != cudaSuccess) return e;
    e = launch_pdl(indexer_multi_gather_kernel, dim3(P, Q, B), dim3(kMqSelThreads), 0, stream,
                   static_cast<const uint32_t*>(keys), cap, seq_len, ratio, Q, k, P,
                   static_cast<const uint32_t*>(ghist), lists, counts);
    if (e != cudaSuccess) return e;
    e = set_smem_once(indexer_multi_select_kernel, sizeof(MqSelSmem));
    if (e != cudaSuccess) return e;
    e = launch_pdl(indexer_multi_select_kernel, dim3(Q, B), dim3(kMqSelThreads), sizeof(MqSelSmem), stream,
                   static_cast<const uint32_t*>(keys), cap, seq_len, ratio, Q, k, P, ghist,
                   static_cast<const uint2*>(lists), static_cast<const uint32_t*>(counts), topk_out);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace csld
