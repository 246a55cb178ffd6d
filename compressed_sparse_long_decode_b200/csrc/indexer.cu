// Lightning indexer + exact top-k.
//
// Source: "DeepSeek-V4: a million-token context that agents can actually use" -- CSA paragraph
// (the lightning indexer, an FP4 ReLU-scored multi-head dot product, picks the top-k
// compressed blocks for each query) and Figure 3 caption; velog.io paper review, "core
// technique 1: CSA" (the indexer scores which compressed entries the query should read).
//
// Score of entry s for one query (4 heads, 64 dims, one key per entry shared by the heads):
//   e_s = sum_h w_h * ReLU(q_h . k_s), q and k both FP4 (E2M1 codes, power-of-two scale / 32).
// The group dots run on the 5th-generation tensor cores as block-scaled FP4 MMAs
// (tcgen05.mma kind::mxf4, M = 128 entries, N = 8, K = 64) with every block scale set to 1, so
// each product of two E2M1 values (a multiple of 1/4, at most 36) and their 32-term sums are
// exact in the fp32 accumulator: the MMA returns I_g / 4 exactly.  B row n holds head n & 3
// over group n >> 2 with the other group's codes zero, so each output column is one group's
// dot.  The fp32 score then follows a fixed operation order (see the ABI header) using the
// true scales, so the selection is reproducible bit for bit; order key = (score, -index).
//
// One kernel (indexer_topk_kernel), grid (chunk, sequence), 16 warps per CTA.  Scoring is
// warp-specialised: warp 12 streams 256-entry tiles of key codes with TMA tensor copies (32-byte
// swizzle, the MMA's canonical K-major layout) and their scales with bulk copies into a 4-stage
// mbarrier ring; warp 13 owns 128 columns of tensor memory and issues two MMAs per tile into
// one of 4 accumulator slots; warpgroups 0..2 take turns reading a slot back (tcgen05.ld, one
// thread per TMEM lane = two entries), forming the 32-bit order keys in shared memory and a
// histogram of their top 11 bits.  The CTA then selects its chunk's top min(k, chunk) -- threshold
// bin from the histogram, one pass to count and collect that bin's candidates, a radix
// select among the candidates only, one pass to emit in index order -- written as a run.  The runs are then merged by a tree inside the same kernel:
// the last CTA of a group of G runs to finish (an atomic arrival counter; nothing ever waits)
// loads the group's runs, selects their top min(k, ...) and publishes one run for the next
// level; the last run is the answer, written in ascending index order and -1 padded.
// Selecting the top k of a union of per-part top-k sets is exact under the total order
// (score desc, index asc), because every global top-k entry is in its part's top k.
#include <cudaTypedefs.h>

#include <mutex>

#include "csld_internal.cuh"
#include "kernels.cuh"
#include "sm100.cuh"

namespace csld {

constexpr int kIdxThreads = 512;
constexpr int kIdxWarps = kIdxThreads / 32;
constexpr int kIdxTile = 256;          // entries per pipeline stage: two 128-row MMAs
constexpr int kIdxStages = 4;
constexpr int kIdxEpiGroups = 3;       // epilogue warpgroups: warps 0..11
constexpr int kIdxProducerWarp = 12;   // issues the tensor / bulk copies
constexpr int kIdxMmaWarp = 13;        // owns the tensor memory, issues the MMAs
constexpr uint32_t kIdxTmemCols = 128; // accumulator slot s = columns 16s..16s+15; scale factors
constexpr uint32_t kIdxSfCol = 64;     // columns 64..71 (A) and 72..79 (B)
constexpr uint32_t kIdxIdesc = idesc_mxf4_m128(8);
constexpr int kIdxMaxChunk = 8192;     // keys a CTA holds (chunk, or runs being merged)
constexpr int kIdxMaxGroup = 64;       // runs merged by one CTA
constexpr int kIdxMaxLevels = 4;
constexpr int kBinShift = 21;          // histogram bin = top 11 bits of the order key
constexpr int kBins = 1 << (32 - kBinShift);
constexpr int kRadixBits = 11;
constexpr int kRadixBins = 1 << kRadixBits;
constexpr int kIdxSmemAlign = 1024;    // swizzled operand tiles start on 1024-byte boundaries

struct IdxSmem {
    union {
        struct {
            uint8_t codes[kIdxStages][kIdxTile * kIkey];   // key codes, K-major 32-byte swizzle
            float scales[kIdxStages][kIdxTile * 2];
        } pipe;                        // key stream ring (scoring)
        struct {
            uint32_t key[kIdxMaxChunk];
            uint16_t pos[kIdxMaxChunk];
        } cand;                        // threshold-bin candidates (selection)
    } u;
    alignas(256) uint8_t bq[8 * kIkey];   // query operand (B): 8 rows x 32 bytes, swizzled
    uint32_t keys[kIdxMaxChunk];       // order keys of the chunk, or of the runs being merged
    uint32_t hist[kBins];              // top-11-bit histogram of keys[]
    uint32_t rhist[kRadixBins];        // radix passes over the candidates
    uint32_t wgt[kIdxWarps], wsel[kIdxWarps], weq[kIdxWarps], wbase[kIdxWarps], weqb[kIdxWarps];
    uint32_t red[2 * kIdxWarps];
    int32_t offs[kIdxMaxGroup + 1];
    float qscale[8];                   // [group*4 + head]
    uint64_t full[kIdxStages];         // stage landed (copies)
    uint64_t empty[kIdxStages];        // stage and accumulator slot consumed (epilogue)
    uint64_t accf[kIdxStages];         // accumulator slot written (MMA commit)
    uint64_t drain;
    uint32_t tmem_base;
    int32_t n_issued, n_mma, fail;
    uint32_t sel[4];                   // bin / threshold results
    uint32_t ncand;
    int32_t last;
};
static_assert(sizeof(((IdxSmem*)0)->u.pipe) <= sizeof(((IdxSmem*)0)->u.cand), "pipe fits the candidate area");

// ------------------------------------------------------------------------------------------
// Block-level helpers (512 threads).
// ------------------------------------------------------------------------------------------
// Radix select among n candidate keys (read through get): the largest `want` (< n), ties on the
// threshold left to the caller (who takes the first take_eq equal keys by position).  The bits
// shared by all candidates are skipped; the rest are resolved 11 bits per pass.
template <typename Get>
__device__ uint32_t radix_select(Get get, int n, int want, uint32_t* hist, uint32_t* sel,
                                 uint32_t* red, uint32_t* take_eq) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    uint32_t kor = 0u, kand = 0xFFFFFFFFu;
    for (int i = tid; i < n; i += blockDim.x) {
        const uint32_t key = get(i);
        kor |= key;
        kand &= key;
    }
    kor = __reduce_or_sync(0xffffffffu, kor);
    kand = __reduce_and_sync(0xffffffffu, kand);
    if (lane == 0) {
        red[warp] = kor;
        red[nw + warp] = kand;
    }
    __syncthreads();
    kor = 0u;
    kand = 0xFFFFFFFFu;
    for (int w = 0; w < nw; ++w) {
        kor |= red[w];
        kand &= red[nw + w];
    }
    __syncthreads();
    const uint32_t diff = kor ^ kand;
    if (diff == 0u) {
        *take_eq = static_cast<uint32_t>(want);
        return kand;
    }
    int top = 31 - __clz(diff);
    uint32_t himask = (top == 31) ? 0u : ~((2u << top) - 1u);
    uint32_t prefix = kand & himask;
    uint32_t remaining = static_cast<uint32_t>(want);
    while (true) {
        const int shift = max(top - (kRadixBits - 1), 0);
        const uint32_t nb = 1u << (top - shift + 1);
        for (uint32_t i = tid; i < nb; i += blockDim.x) hist[i] = 0u;
        __syncthreads();
        for (int i = tid; i < n; i += blockDim.x) {
            const uint32_t key = get(i);
            if (((key ^ prefix) & himask) == 0u) atomicAdd(&hist[(key >> shift) & (nb - 1u)], 1u);
        }
        __syncthreads();
        const uint32_t per = (nb + blockDim.x - 1) / blockDim.x;
        uint32_t tot = 0u;
        for (uint32_t q = 0; q < per; ++q) {
            const int d = static_cast<int>(nb) - 1 - static_cast<int>(tid * per + q);
            if (d >= 0) tot += hist[d];
        }
        uint32_t incl = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) red[warp] = incl;
        __syncthreads();
        uint32_t wb = 0u;
        for (int w = 0; w < warp; ++w) wb += red[w];
        incl += wb;
        const uint32_t excl = incl - tot;
        if (excl < remaining && incl >= remaining) {
            uint32_t run = excl;
            for (uint32_t q = 0; q < per; ++q) {
                const int d = static_cast<int>(nb) - 1 - static_cast<int>(tid * per + q);
                if (d < 0) break;
                if (run + hist[d] >= remaining) {
                    sel[0] = static_cast<uint32_t>(d);
                    sel[1] = remaining - run;
                    break;
                }
                run += hist[d];
            }
        }
        __syncthreads();
        prefix |= sel[0] << shift;
        himask |= (nb - 1u) << shift;
        remaining = sel[1];
        __syncthreads();
        if (shift == 0) break;
        top = shift - 1;
    }
    *take_eq = remaining;
    return prefix;
}

// Selects the top `want` of sm.keys[0..n) under (key desc, position asc) and emits them in
// position order: emit(out_pos, position).  Requires sm.hist = histogram of key >> kBinShift.
template <typename Emit>
__device__ void select_emit(IdxSmem& sm, int n, int want, Emit emit) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t lt = (1u << lane) - 1u;
    const int seg = ((n + kIdxWarps - 1) / kIdxWarps + 31) & ~31;
    const int i0 = min(n, warp * seg), i1 = min(n, i0 + seg);
    if (want >= n) {                                   // everything is selected
        for (int base = i0; base < i1; base += 32)
            if (base + lane < i1) emit(base + lane, base + lane);
        __syncthreads();
        return;
    }
    // 1) the bin holding the want-th largest key (thread t owns bins 2047-4t .. 2044-4t)
    {
        uint32_t c[4], tot = 0u;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            c[q] = sm.hist[kBins - 1 - 4 * tid - q];
            tot += c[q];
        }
        uint32_t incl = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) sm.red[warp] = incl;
        if (tid == 0) sm.ncand = 0u;
        __syncthreads();
        uint32_t wb = 0u;
        for (int w = 0; w < warp; ++w) wb += sm.red[w];
        incl += wb;
        const uint32_t excl = incl - tot;
        const uint32_t W = static_cast<uint32_t>(want);
        if (excl < W && incl >= W) {
            uint32_t run = excl;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                if (run + c[q] >= W) {
                    sm.sel[0] = static_cast<uint32_t>(kBins - 1 - 4 * tid - q);   // bin beta
                    sm.sel[1] = W - run;                                          // wanted inside it
                    break;
                }
                run += c[q];
            }
        }
        if (tid < kIdxWarps) {
            sm.wsel[tid] = 0u;
            sm.weq[tid] = 0u;
        }
        __syncthreads();
    }
    const uint32_t beta = sm.sel[0], need = sm.sel[1];
    // 2) pass 1: per-warp count above the bin; collect the bin's candidates with positions
    uint32_t gt = 0u;
    for (int base = i0; base < i1; base += 32) {
        const int i = base + lane;
        const uint32_t key = i < i1 ? sm.keys[i] : 0u;
        const uint32_t bin = key >> kBinShift;
        gt += __popc(__ballot_sync(0xffffffffu, i < i1 && bin > beta));
        const uint32_t cm = __ballot_sync(0xffffffffu, i < i1 && bin == beta);
        if (cm) {
            uint32_t slot = 0u;
            if (lane == 0) slot = atomicAdd(&sm.ncand, static_cast<uint32_t>(__popc(cm)));
            slot = __shfl_sync(0xffffffffu, slot, 0);
            if (i < i1 && bin == beta) {
                const uint32_t at = slot + __popc(cm & lt);
                sm.u.cand.key[at] = key;
                sm.u.cand.pos[at] = static_cast<uint16_t>(i);
            }
        }
    }
    if (lane == 0) sm.wgt[warp] = gt;
    __syncthreads();
    // 3) exact threshold among the candidates
    const int P = static_cast<int>(sm.ncand);
    uint32_t thr = 0u, take_eq = static_cast<uint32_t>(P);
    if (static_cast<int>(need) < P)
        thr = radix_select([&](int c) { return sm.u.cand.key[c]; }, P, static_cast<int>(need), sm.rhist, sm.sel + 2,
                           sm.red, &take_eq);
    // 4) per-warp counts of selected candidates (above the threshold, equal to it)
    for (int c = tid; c < P; c += blockDim.x) {
        const uint32_t key = sm.u.cand.key[c];
        const int w = sm.u.cand.pos[c] / seg;
        if (key > thr) atomicAdd(&sm.wsel[w], 1u);
        else if (key == thr) atomicAdd(&sm.weq[w], 1u);
    }
    __syncthreads();
    if (warp == 0) {
        const uint32_t e = lane < kIdxWarps ? sm.weq[lane] : 0u;
        uint32_t ei = e;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, ei, o);
            if (lane >= o) ei += y;
        }
        const uint32_t eb = ei - e;
        const uint32_t tw = eb >= take_eq ? 0u : min(e, take_eq - eb);
        const uint32_t tk = (lane < kIdxWarps ? sm.wgt[lane] + sm.wsel[lane] : 0u) + tw;
        uint32_t ti = tk;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, ti, o);
            if (lane >= o) ti += y;
        }
        if (lane < kIdxWarps) {
            sm.wbase[lane] = ti - tk;
            sm.weqb[lane] = eb;
        }
    }
    __syncthreads();
    // 5) pass 2: emit in position order
    uint32_t pos = sm.wbase[warp], eq_seen = sm.weqb[warp];
    for (int base = i0; base < i1; base += 32) {
        const int i = base + lane;
        const uint32_t key = i < i1 ? sm.keys[i] : 0u;
        const uint32_t bin = key >> kBinShift;
        const bool inb = i < i1 && bin == beta;
        const bool veq = inb && key == thr;
        const uint32_t em = __ballot_sync(0xffffffffu, veq);
        const bool take = (i < i1 && bin > beta) || (inb && key > thr) || (veq && eq_seen + __popc(em & lt) < take_eq);
        const uint32_t tm = __ballot_sync(0xffffffffu, take);
        if (take) emit(pos + __popc(tm & lt), i);
        pos += __popc(tm);
        eq_seen += __popc(em);
    }
    __syncthreads();
}

// ------------------------------------------------------------------------------------------
// Workspace layout of the merge tree.
// ------------------------------------------------------------------------------------------
struct IdxTree {
    int levels;                        // run levels that are stored (the final run is not)
    int n_runs[kIdxMaxLevels + 1];     // runs per sequence at each level (level 0 = chunks)
    int rcap[kIdxMaxLevels + 1];       // candidates a run of each level can hold
    uint32_t* keys[kIdxMaxLevels];     // [B][n_runs[l]][rcap[l]]
    int32_t* idx[kIdxMaxLevels];
    int32_t* cnt[kIdxMaxLevels];       // [B][n_runs[l]]
    int32_t* ctr[kIdxMaxLevels + 1];   // arrival counters of level l runs, [B][n_runs[l]]
    int group;
};

static size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

// Level-0 runs hold min(k, chunk) candidates; merged runs hold up to k.
static IdxTree tree_layout(int B, int n_chunks, int kc, int k, int group, uint8_t* base, size_t* bytes) {
    IdxTree t{};
    t.group = group;
    t.n_runs[0] = n_chunks;
    t.rcap[0] = kc;
    for (int i = 1; i <= kIdxMaxLevels; ++i) t.rcap[i] = k;
    int l = 0;
    while (t.n_runs[l] > 1 && l < kIdxMaxLevels) {
        t.n_runs[l + 1] = (t.n_runs[l] + group - 1) / group;
        ++l;
    }
    t.levels = l;  // levels 0..l-1 store runs; level l has exactly one run (the answer)
    size_t off = 0;
    for (int i = 0; i < t.levels; ++i) {
        const size_t slots = (size_t)B * t.n_runs[i] * t.rcap[i];
        t.keys[i] = reinterpret_cast<uint32_t*>(base ? base + off : nullptr);
        off += up256(slots * 4);
        t.idx[i] = reinterpret_cast<int32_t*>(base ? base + off : nullptr);
        off += up256(slots * 4);
        t.cnt[i] = reinterpret_cast<int32_t*>(base ? base + off : nullptr);
        off += up256((size_t)B * t.n_runs[i] * 4);
    }
    for (int i = 1; i <= t.levels; ++i) {
        t.ctr[i] = reinterpret_cast<int32_t*>(base ? base + off : nullptr);
        off += up256((size_t)B * t.n_runs[i] * 4);
    }
    *bytes = off;
    return t;
}

// ------------------------------------------------------------------------------------------
// The kernel.
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kIdxThreads, 2) indexer_topk_kernel(
    const __grid_constant__ CUtensorMap kmap, const float* __restrict__ iscales, int64_t cap,
    const int32_t* __restrict__ seq_len, int ratio, const float* __restrict__ q_idx,
    const float* __restrict__ head_w, int chunk, int kc, int k, IdxTree tree,
    int32_t* __restrict__ topk_out, int32_t* err) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    IdxSmem& sm = *reinterpret_cast<IdxSmem*>(
        smem_raw + ((kIdxSmemAlign - (smem_u32(smem_raw) & (kIdxSmemAlign - 1))) & (kIdxSmemAlign - 1)));
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = blockIdx.y, ch = blockIdx.x;

    int64_t n_b = seq_len[b];
    n_b = n_b < 0 ? 0 : n_b / ratio;
    if (n_b > cap) n_b = cap;
    const int64_t c0 = (int64_t)ch * chunk;
    const int cn = static_cast<int>(max64(0, min64(chunk, n_b - c0)));

    for (int i = tid; i < kBins; i += blockDim.x) sm.hist[i] = 0u;
    bool chunk_ok = true;
    if (cn > 0) {
        const int n_tiles = (cn + kIdxTile - 1) / kIdxTile;
        volatile int32_t* fail = &sm.fail;
        if (tid == 0) {
            for (int s = 0; s < kIdxStages; ++s) {
                mbar_init(&sm.full[s], 1);
                mbar_init(&sm.empty[s], 4);          // the 4 warps of the epilogue warpgroup
                mbar_init(&sm.accf[s], 1);
            }
            mbar_init(&sm.drain, 1);
            sm.fail = 0;
            sm.n_issued = 0;
            sm.n_mma = 0;
            fence_barrier_init();
        }
        if (warp == kIdxMmaWarp) {
            tmem_alloc(&sm.tmem_base, kIdxTmemCols);
            tmem_relinquish();
        }
        if (warp == kIdxProducerWarp && lane == 0) tma_prefetch_map(&kmap);
        // --- query operand: FP4 codes in the MMA's B layout (8 rows x 32 bytes, 32-byte swizzle)
        // Row n is head n & 3 over group n >> 2; the row's other 32-element group is zero, so
        // every output column is one exact group dot.  Thread t writes bytes 4j..4j+3 of row n.
        if (tid < 64) {
            const int n = tid >> 3, j = tid & 7, h = n & 3, grp = n >> 2;
            const float* qv = q_idx + ((size_t)b * kIdxHeads + h) * kIdxDim;
            float amax = 0.f;
            for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(qv[32 * grp + i]));
            const float sg = fp4_group_scale(amax);
            const float inv = 1.0f / sg;   // exact: a power of two
            uint32_t word = 0u;
            if ((j >> 2) == grp) {
#pragma unroll
                for (int i = 0; i < 8; ++i) word |= e2m1_code(qv[8 * j + i] * inv) << (4 * i);
            }
            const int half = (j >> 2) ^ ((n >> 2) & 1);
            *reinterpret_cast<uint32_t*>(sm.bq + n * kIkey + half * 16 + (j & 3) * 4) = word;
            if (j == 0) sm.qscale[grp * 4 + h] = sg;
            fence_proxy_async_smem();
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        const uint32_t tmem = sm.tmem_base;
        if (warp < 4) {   // unit block-scale factors (UE8M0 0x7F = 2^0) for A and B, every lane
            tmem_st_32x32b_x8_fill(tmem + ((32u * warp) << 16) + kIdxSfCol, 0x7F7F7F7Fu);
            tmem_st_32x32b_x8_fill(tmem + ((32u * warp) << 16) + kIdxSfCol + 8, 0x7F7F7F7Fu);
            tmem_st_wait();
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        const float* sbase = iscales + ((size_t)b * cap + (size_t)c0) * 2;
        if (warp == kIdxProducerWarp) {
            // --- producer: key tile (TMA, swizzled) + its scales (bulk copy) per stage -------
            if (lane == 0) {
                int t = 0;
                for (; t < n_tiles; ++t) {
                    const int s = t % kIdxStages;
                    if (*fail) break;
                    if (t >= kIdxStages && !mbar_wait(&sm.empty[s], ((t / kIdxStages) - 1) & 1)) break;
                    const int nt = min(kIdxTile, cn - t * kIdxTile);
                    const uint32_t sb = static_cast<uint32_t>((nt + 1) & ~1) * 8u;   // cap is even
                    mbar_arrive_expect_tx(&sm.full[s], kIdxTile * kIkey + sb);
                    tma_load_3d(sm.u.pipe.codes[s], &kmap, 0, static_cast<int>(c0) + t * kIdxTile, b, &sm.full[s]);
                    bulk_g2s(sm.u.pipe.scales[s], sbase + (size_t)t * kIdxTile * 2, sb, &sm.full[s]);
                }
                sm.n_issued = t;
                if (t < n_tiles) *fail = 1;
            }
        } else if (warp == kIdxMmaWarp) {
            // --- MMA issuer: two 128-row block-scaled FP4 MMAs per tile into accumulator slot s
            if (lane == 0) {
                const uint64_t bdesc = smem_desc_kmajor_sw32(sm.bq);
                const uint32_t sfa = tmem + kIdxSfCol, sfb = tmem + kIdxSfCol + 8;
                int t = 0;
                for (; t < n_tiles; ++t) {
                    const int s = t % kIdxStages;
                    if (*fail || !mbar_wait(&sm.full[s], (t / kIdxStages) & 1)) break;
                    tc_fence_after();
                    const uint32_t d = tmem + 16u * static_cast<uint32_t>(s);
                    umma_mxf4(d, smem_desc_kmajor_sw32(sm.u.pipe.codes[s]), bdesc, kIdxIdesc, sfa, sfb, 0u);
                    umma_mxf4(d + 8u, smem_desc_kmajor_sw32(sm.u.pipe.codes[s] + 128 * kIkey), bdesc, kIdxIdesc,
                              sfa, sfb, 0u);
                    umma_commit(&sm.accf[s]);
                }
                sm.n_mma = t;
                if (t < n_tiles) *fail = 1;
            }
        } else if (warp < 4 * kIdxEpiGroups) {
            // --- epilogue: warpgroup wg finishes tiles wg, wg + 3, ...; thread = TMEM lane m
            // holds entries m and 128 + m of the tile: columns 0..3 / 4..7 their group-0 /
            // group-1 dots of heads 0..3 (8..15 for entry 128 + m), each exactly I_g / 4.
            const int wg = warp >> 2, quad = warp & 3;
            const int m = 32 * quad + lane;
            const uint32_t lane_addr = tmem + ((32u * quad) << 16);
            float qsc[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) qsc[i] = sm.qscale[i];
            const float w0 = head_w[b * kIdxHeads + 0], w1 = head_w[b * kIdxHeads + 1];
            const float w2 = head_w[b * kIdxHeads + 2], w3 = head_w[b * kIdxHeads + 3];
            for (int t = wg; t < n_tiles; t += kIdxEpiGroups) {
                const int s = t % kIdxStages;
                const bool landed = !*fail && mbar_wait(&sm.accf[s], (t / kIdxStages) & 1);
                if (!__all_sync(0xffffffffu, landed)) {
                    if (lane == 0) *fail = 1;
                    break;
                }
                tc_fence_after();
                uint32_t r[16];
                tmem_ld_32x32b_x16(lane_addr + 16u * static_cast<uint32_t>(s), r);
                tmem_ld_wait();
                const float2* ss = reinterpret_cast<const float2*>(sm.u.pipe.scales[s]);
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    const int e = 128 * hf + m;
                    const float2 ks = ss[e];
                    float rr[4];
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        // d = fma(I1, s1, I0*s0) with s_g = (qscale_g * kscale_g) * 0.25
                        const float i0 = __fmul_rn(__uint_as_float(r[8 * hf + h]), 4.0f);
                        const float i1 = __fmul_rn(__uint_as_float(r[8 * hf + 4 + h]), 4.0f);
                        const float s0 = __fmul_rn(__fmul_rn(qsc[h], ks.x), 0.25f);
                        const float s1 = __fmul_rn(__fmul_rn(qsc[4 + h], ks.y), 0.25f);
                        const float d = __fmaf_rn(i1, s1, __fmul_rn(i0, s0));
                        rr[h] = d > 0.f ? d : 0.f;
                    }
                    float sc = __fmul_rn(w0, rr[0]);
                    sc = __fmaf_rn(w1, rr[1], sc);
                    sc = __fmaf_rn(w2, rr[2], sc);
                    sc = __fmaf_rn(w3, rr[3], sc);
                    const int li = t * kIdxTile + e;
                    if (li < cn) {
                        const uint32_t key = score_key(sc);
                        sm.keys[li] = key;
                        atomicAdd(&sm.hist[key >> kBinShift], 1u);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.empty[s]);   // stage s and accumulator slot s free
            }
        }
        tc_fence_before();
        __syncthreads();
        chunk_ok = (sm.fail == 0);
        if (!chunk_ok) {
            // A copy or an MMA did not complete in time: record it, let the copies in flight
            // land and the MMAs in flight finish (bounded waits) before the shared and tensor
            // memory are reused, and publish this chunk as empty so the merge tree completes.
            if (warp == kIdxMmaWarp && lane == 0) {
                dev_error(err, CSLD_DEVERR_TIMEOUT);
                for (int t = sm.n_mma; t < sm.n_issued; ++t)
                    (void)mbar_wait(&sm.full[t % kIdxStages], (t / kIdxStages) & 1);
                umma_commit(&sm.drain);
                (void)mbar_wait(&sm.drain, 0);
            }
            __syncthreads();
        }
        if (warp == kIdxMmaWarp) {
            tc_fence_after();
            tmem_dealloc(tmem, kIdxTmemCols);
        }
    }
    __syncthreads();
    // --- selection and the merge tree ------------------------------------------------------
    int n = (cn > 0 && chunk_ok) ? cn : 0;   // a timed-out chunk publishes nothing
    int level = 0, run = ch;
    const uint32_t* child_idx = nullptr;     // merge levels: indices stay in the children runs
    for (;;) {
        const int n_runs = tree.n_runs[level];
        const bool final_run = (n_runs == 1);
        const int want = min(final_run ? k : tree.rcap[level], n);
        const size_t rb = final_run ? 0 : ((size_t)b * n_runs + run) * tree.rcap[level];
        int32_t* out = topk_out + (size_t)b * k;
        if (level == 0) {
            // chunk level: the entry index of position i is c0 + i
            if (final_run) {
                select_emit(sm, n, want, [&](int p, int i) { out[p] = static_cast<int32_t>(c0 + i); });
            } else {
                uint32_t* okeys = tree.keys[0] + rb;
                int32_t* oidx = tree.idx[0] + rb;
                select_emit(sm, n, want, [&](int p, int i) {
                    okeys[p] = sm.keys[i];
                    oidx[p] = static_cast<int32_t>(c0 + i);
                });
            }
        } else {
            // merge levels: the entry indices stay in the children runs (L2).  The ordered pass
            // records positions only; the indices are then fetched together, so their loads
            // overlap instead of costing one round trip per 32 keys.
            select_emit(sm, n, want, [&](int p, int i) { sm.rhist[p] = static_cast<uint32_t>(i); });
            const int rcc = tree.rcap[level - 1];
            for (int p = tid; p < want; p += blockDim.x) {
                const int i = static_cast<int>(sm.rhist[p]);
                int lo = 0, hi = kIdxMaxGroup - 1;           // child c with offs[c] <= i < offs[c+1]
                while (lo < hi) {
                    const int mid = (lo + hi + 1) >> 1;
                    if (sm.offs[mid] <= i) lo = mid;
                    else hi = mid - 1;
                }
                const int32_t idx = __ldcg(reinterpret_cast<const int32_t*>(child_idx) + (size_t)lo * rcc + (i - sm.offs[lo]));
                if (final_run) {
                    out[p] = idx;
                } else {
                    tree.keys[level][rb + p] = sm.keys[i];
                    tree.idx[level][rb + p] = idx;
                }
            }
            __syncthreads();
        }
        if (final_run) {
            for (int i = want + tid; i < k; i += blockDim.x) out[i] = -1;
            return;
        }
        if (tid == 0) tree.cnt[level][(size_t)b * n_runs + run] = want;
        // arrive at the parent; the last child to arrive carries on with the merge
        const int parent = run / tree.group;
        const int n_par = tree.n_runs[level + 1];
        const int children = min(tree.group, n_runs - parent * tree.group);
        __syncthreads();
        if (tid == 0) {
            __threadfence();
            int32_t* ctr = tree.ctr[level + 1] + (size_t)b * n_par + parent;
            const int old = atomicAdd(ctr, 1);
            sm.last = (old == children - 1);
            if (sm.last) {
                *ctr = 0;          // leave the counter ready for the next call
                __threadfence();
            }
        }
        __syncthreads();
        if (!sm.last) return;
        // load the children runs' keys (published by other CTAs: read through L2) and rebuild
        // the histogram; their indices are read from L2 when emitting
        if (tid == 0) {
            int acc = 0;
            for (int c = 0; c < children; ++c) {
                sm.offs[c] = acc;
                acc += __ldcg(tree.cnt[level] + (size_t)b * n_runs + parent * tree.group + c);
            }
            sm.offs[children] = acc;
            for (int c = children + 1; c <= kIdxMaxGroup; ++c) sm.offs[c] = 1 << 30;   // > any position
        }
        for (int i = tid; i < kBins; i += blockDim.x) sm.hist[i] = 0u;
        __syncthreads();
        const size_t child0 = ((size_t)b * n_runs + (size_t)parent * tree.group) * tree.rcap[level];
        const int rc = tree.rcap[level];
        for (int base = 0; base < children * rc; base += 8 * blockDim.x) {
            uint32_t kv[8];
            int dst[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int flat = base + u * blockDim.x + tid;     // child c, position i
                const int c = flat / rc, i = flat - c * rc;
                dst[u] = -1;
                if (c < children && i < sm.offs[c + 1] - sm.offs[c]) {
                    kv[u] = __ldcg(tree.keys[level] + child0 + flat);
                    dst[u] = sm.offs[c] + i;
                }
            }
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (dst[u] >= 0) {
                    sm.keys[dst[u]] = kv[u];
                    atomicAdd(&sm.hist[kv[u] >> kBinShift], 1u);
                }
        }
        child_idx = reinterpret_cast<const uint32_t*>(tree.idx[level] + child0);
        n = sm.offs[children];
        __syncthreads();
        ++level;
        run = parent;
    }
}

IndexerPlan indexer_plan(int B, int64_t cap, int k, int num_sms) {
    IndexerPlan p;
    int chunk = kIdxMaxChunk;
    while (chunk > 1024 && (int64_t)B * ((cap + chunk - 1) / chunk) < num_sms) chunk >>= 1;
    p.chunk = chunk;
    const int64_t nc = (cap + chunk - 1) / chunk;
    p.n_chunks = static_cast<int>(nc < 1 ? 1 : nc);
    p.kc = k < chunk ? k : chunk;
    int group = kIdxMaxChunk / k;                 // merged runs hold up to k candidates
    if (group > kIdxMaxGroup) group = kIdxMaxGroup;
    if (group < 2) group = 2;
    p.group = group;
    size_t bytes = 0;
    IdxTree t = tree_layout(B, p.n_chunks, p.kc, k, group, nullptr, &bytes);
    p.levels_ok = (t.n_runs[t.levels] == 1);
    p.ws_bytes = bytes;
    return p;
}

// cuTensorMapEncodeTiled from the driver (through the runtime, so nothing links libcuda).
static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

cudaError_t launch_indexer(const uint8_t* ikeys, const float* iscales, int64_t cap,
                           const int32_t* seq_len, int ratio, const float* q_idx,
                           const float* head_w, int B, int k, int32_t* topk_out, void* ws,
                           const IndexerPlan& plan, int32_t* err, cudaStream_t stream) {
    size_t bytes = 0;
    IdxTree tree = tree_layout(B, plan.n_chunks, plan.kc, k, plan.group, static_cast<uint8_t*>(ws), &bytes);
    // Key codes as a 3-D byte tensor [B][cap][32]; one box = one stage of 256 entries.  Rows
    // past cap read as zeros (their scores are never used).
    PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
    if (encode == nullptr) return cudaErrorNotSupported;
    CUtensorMap kmap;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kIkey), static_cast<cuuint64_t>(cap), static_cast<cuuint64_t>(B)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(kIkey), static_cast<cuuint64_t>(cap) * kIkey};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(kIkey), static_cast<cuuint32_t>(kIdxTile), 1u};
    const cuuint32_t estr[3] = {1u, 1u, 1u};
    if (encode(&kmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(ikeys), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    const size_t smem = sizeof(IdxSmem) + kIdxSmemAlign;
    cudaError_t e = set_smem_once(indexer_topk_kernel, smem);
    if (e != cudaSuccess) return e;
    dim3 grid(plan.n_chunks, B);
    indexer_topk_kernel<<<grid, kIdxThreads, smem, stream>>>(kmap, iscales, cap, seq_len, ratio,
                                                             q_idx, head_w, plan.chunk, plan.kc, k,
                                                             tree, topk_out, err);
    return cudaGetLastError();
}

}  // namespace csld
