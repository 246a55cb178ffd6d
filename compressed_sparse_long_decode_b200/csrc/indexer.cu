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
// Scoring (score_setup + score_run, shared by both kernels below) is warp-specialised over 16
// warps: warp 12 streams 256-entry tiles of key codes into an mbarrier ring with 1-D bulk
// copies -- the cache stores the codes pre-swizzled (32-byte swizzle, the MMA's canonical
// K-major layout), so they land ready to use -- together with their scales, several tiles per
// copy; warp 13 owns the tensor memory and issues two MMAs per tile into one of the
// accumulator slots; warpgroups 0..2 take turns reading a slot back (tcgen05.ld, one thread
// per TMEM lane = two entries), forming the 32-bit order keys in shared memory and a histogram
// of their top 11 bits.
//
// Selection, when the whole grid can be resident (indexer_topk_coop_kernel, cooperative
// launch): each sequence is split into `units` ranges, one CTA each, and the CTAs of a sequence
// run an exact select together.  They add their histograms into the sequence's global
// histogram, each re-read it until its bins account for every key of the sequence (every wait
// is bounded), and each derive the same threshold bin.  When that bin holds at most kListMax keys, every CTA appends its keys in
// the bin to a list of self-announcing slots, then reads the whole list as it fills and finds
// the exact threshold key with three radix levels; otherwise two more histogram rounds over
// the next 11 and 10 key bits (and arrival-counter barriers) give it.  Either way every CTA learns how many
// selected entries precede its range (ties go to the lowest indices) and writes its own in
// ascending index order.
//
// Otherwise (indexer_topk_kernel): each CTA selects its chunk's top min(k, chunk) -- threshold
// bin from the histogram, the bin's candidates collected, a radix select among them, an emit in
// index order -- written as a run, and the runs are merged by a tree inside the same kernel:
// the last CTA of a group of G runs to finish (an atomic arrival counter; nothing ever waits)
// loads the group's runs, selects their top min(k, ...) and publishes one run for the next
// level; the last run is the answer, written in ascending index order and -1 padded.
// Selecting the top k of a union of per-part top-k sets is exact under the total order
// (score desc, index asc), because every global top-k entry is in its part's top k.
#include <cudaTypedefs.h>

#include <atomic>
#include <mutex>

#include "csld_internal.cuh"
#include "kernels.cuh"
#include "sm100.cuh"

namespace csld {

constexpr int kIdxThreads = 512;
constexpr int kIdxWarps = kIdxThreads / 32;
constexpr int kIdxTile = 256;          // entries per pipeline stage: two 128-row MMAs
constexpr int kIdxStages = 4;          // ring depth of the merge-tree kernel (shares the candidate area)
constexpr int kCoopStages = 12;        // ring depth of the cooperative kernel (one CTA per SM)
constexpr int kCoopGroup = 4;          // tiles per key copy in the cooperative kernel (32 KB of codes)
constexpr int kMaxStages = 12;
constexpr int kIdxEpiGroups = 3;       // epilogue warpgroups: warps 0..11
constexpr int kIdxProducerWarp = 12;   // issues the tensor / bulk copies
constexpr int kIdxMmaWarp = 13;        // owns the tensor memory, issues the MMAs
// Tensor memory: accumulator slot s = columns 16s..16s+15; the last 16 allocated columns hold
// the unit scale factors (8 for A, 8 for B).  128 columns for the 4-slot ring, 256 for 12.
constexpr uint32_t kIdxIdesc = idesc_mxf4_m128(8);
constexpr int kIdxMaxChunk = 8192;     // keys a merge-tree CTA holds (chunk, or runs being merged)
constexpr int kCoopMaxRange = 16384;   // keys a cooperative CTA holds
constexpr int kIdxMaxGroup = 64;       // runs merged by one CTA
constexpr int kIdxMaxLevels = 4;
constexpr int kBinShift = 21;          // histogram bin = top 11 bits of the order key
constexpr int kBins = 1 << (32 - kBinShift);
constexpr int kRadixBits = 11;
constexpr int kRadixBins = 1 << kRadixBits;
constexpr int kIdxSmemAlign = 1024;    // swizzled operand tiles start on 1024-byte boundaries
constexpr int kCoopSeqWords = 2 * kBins + 1024;   // per sequence: three levels of histograms
constexpr int kListMax = 8192;       // candidates a sequence's list holds (cooperative fast path)

// Scoring control block: query operand, ring barriers, tensor-memory base, progress.
struct ScoreCtl {
    alignas(256) uint8_t bq[8 * kIkey];   // query operand (B): 8 rows x 32 bytes, swizzled
    float qscale[8];                   // [group*4 + head]
    uint64_t full[kMaxStages];         // stage landed (copies)
    uint64_t empty[kMaxStages];        // stage and accumulator slot consumed (epilogue)
    uint64_t accf[kMaxStages];         // accumulator slot written (MMA commit)
    uint64_t drain;
    uint32_t tmem_base;
    int32_t n_issued, n_mma, fail;
};

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
    ScoreCtl ctl;
    uint32_t keys[kIdxMaxChunk];       // order keys of the chunk, or of the runs being merged
    uint32_t hist[kBins];              // top-11-bit histogram of keys[]
    uint32_t rhist[kRadixBins];        // radix passes over the candidates
    uint32_t red[3 * kIdxWarps];
    int32_t offs[kIdxMaxGroup + 1];
    uint32_t sel[4];                   // bin / threshold results
    int32_t last;
};
static_assert(sizeof(((IdxSmem*)0)->u.pipe) <= sizeof(((IdxSmem*)0)->u.cand), "pipe fits the candidate area");

struct CoopSmem {
    uint8_t codes[kCoopStages][kIdxTile * kIkey];
    float scales[kCoopStages][kIdxTile * 2];
    ScoreCtl ctl;
    uint32_t keys[kCoopMaxRange];      // order keys of this CTA's range
    uint32_t stepmax[kCoopMaxRange / 32 + 8];   // largest key of each aligned 32-key step
    uint32_t hist[kBins];              // this CTA's histograms of radix levels 1, 2, 3
    uint32_t hist2[kBins];
    uint32_t hist3[1024];
    uint32_t red[3 * kIdxWarps];
    uint32_t sel[4];
    int32_t fail;
};
static_assert(sizeof(((CoopSmem*)0)->codes) >= kCoopMaxRange * 4, "candidate regions fit the idle copy ring");

// ------------------------------------------------------------------------------------------
// Block-level helpers (512 threads).
// ------------------------------------------------------------------------------------------
// Histogram increment with the lanes of a warp that hit the same bin combined into one atomic
// (the keys being merged crowd into few bins).  Every lane of the warp must call it.
__device__ __forceinline__ void hist_add(uint32_t* hist, uint32_t bin, bool valid) {
    const uint32_t same = __match_any_sync(0xffffffffu, valid ? bin : 0xFFFFFFFFu);
    const int lane = threadIdx.x & 31;
    if (valid && lane == __ffs(same) - 1) atomicAdd(&hist[bin], static_cast<uint32_t>(__popc(same)));
}

// Exact threshold among n keys that share their top 11 bits (prefix): the want-th largest key,
// and in *take_eq how many keys equal to it are taken.  Three radix levels of 8, 8 and 5 bits
// over bits 20..0.  A level is one histogram pass by the whole block (plain shared atomics:
// warp-level match_any aggregation measured slower on keys this spread) and a scan of the
// 256 bins by warp 0, which also clears the other histogram buffer for the next level: two CTA
// barriers a level.
// hist holds 512 words; hist[0..255] must be zero on entry.  sel: 2 words of shared scratch.
__device__ uint32_t list_select(const uint32_t* keys, int n, uint32_t want, uint32_t prefix, uint32_t* hist,
                                uint32_t* sel, uint32_t* take_eq) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint32_t himask = 0xFFFFFFFFu << kBinShift;
    uint32_t remaining = want;
#pragma unroll 1
    for (int lv = 0; lv < 3; ++lv) {
        const int shift = lv == 0 ? 13 : (lv == 1 ? 5 : 0);
        const uint32_t dmask = lv == 2 ? 31u : 255u;
        uint32_t* h = hist + 256 * (lv & 1);
        for (int i = tid; i < n; i += blockDim.x) {
            const uint32_t key = keys[i];
            if ((key & himask) == prefix) atomicAdd(&h[(key >> shift) & dmask], 1u);
        }
        __syncthreads();
        if (warp == 0) {
            uint32_t c[8], tot = 0u;   // lane l: digits 255 - 8l down to 248 - 8l
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                c[q] = h[255 - 8 * lane - q];
                tot += c[q];
            }
            uint32_t incl = tot;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            const uint32_t excl = incl - tot;
            if (excl < remaining && incl >= remaining) {
                uint32_t run = excl;
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    if (run + c[q] >= remaining) {
                        sel[0] = static_cast<uint32_t>(255 - 8 * lane - q);
                        sel[1] = remaining - run;
                        break;
                    }
                    run += c[q];
                }
            }
            uint32_t* o = hist + 256 * ((lv + 1) & 1);
#pragma unroll
            for (int q = 0; q < 8; ++q) o[8 * lane + q] = 0u;
        }
        __syncthreads();
        prefix |= sel[0] << shift;
        remaining = sel[1];
        himask |= dmask << shift;
    }
    *take_eq = remaining;
    return prefix;
}

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

// Warp-level exclusive prefix over the 16 warps of the block: v is the warp's value (uniform in
// the warp); returns the sum over lower warps, *total the block's sum.  red: kIdxWarps words
// not touched by anyone else until the next barrier.
__device__ __forceinline__ uint32_t warp_excl_scan(uint32_t v, uint32_t* red, uint32_t* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) red[warp] = v;
    __syncthreads();
    uint32_t before = 0u, all = 0u;
#pragma unroll
    for (int w = 0; w < kIdxWarps; ++w) {
        const uint32_t r = red[w];
        before += (w < warp) ? r : 0u;
        all += r;
    }
    *total = all;
    return before;
}

// Sums a and e over the 512 threads of the block (every thread gets both sums).  red: 32 words
// no one else uses until the trailing barrier.
__device__ __forceinline__ void block_sum2(uint32_t a, uint32_t e, uint32_t* red, uint32_t* A, uint32_t* E) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    a = __reduce_add_sync(0xffffffffu, a);
    e = __reduce_add_sync(0xffffffffu, e);
    if (lane == 0) {
        red[warp] = a;
        red[kIdxWarps + warp] = e;
    }
    __syncthreads();
    uint32_t sa = 0u, se = 0u;
#pragma unroll
    for (int w = 0; w < kIdxWarps; ++w) {
        sa += red[w];
        se += red[kIdxWarps + w];
    }
    *A = sa;
    *E = se;
    __syncthreads();
}


// Selects the top `want` of sm.keys[0..n) under (key desc, position asc) and emits them in
// position order: emit(out_pos, position).  Requires sm.hist = histogram of key >> kBinShift.
// Warp w owns positions 512w .. 512w+511, read 32 at a time (lane = position mod 32), so warp
// order then step order then lane order is position order; every count comes from ballots and
// two prefix sums over the 16 warps: no atomics and no dependent round trips per key.
template <typename Emit>
__device__ void select_emit(IdxSmem& sm, int n, int want, Emit emit) {
    constexpr int kSeg = kIdxMaxChunk / kIdxWarps;     // 512 positions per warp
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t lt = (1u << lane) - 1u;
    const int i0 = warp * kSeg;
    const int steps = max(0, min(kSeg, n - i0) + 31) >> 5;
    if (want >= n) {                                   // everything is selected
        for (int s = 0; s < steps; ++s) {
            const int i = i0 + 32 * s + lane;
            if (i < n) emit(i, i);
        }
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
        uint32_t all;
        const uint32_t wb = warp_excl_scan(__shfl_sync(0xffffffffu, incl, 31), sm.red, &all);
        const uint32_t excl = wb + incl - tot;
        const uint32_t W = static_cast<uint32_t>(want);
        if (excl < W && excl + tot >= W) {
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
        __syncthreads();
    }
    const uint32_t beta = sm.sel[0], need = sm.sel[1];
    // 2) per warp: keys above the bin and keys in it; the bin's candidates are then written
    //    compactly in position order
    uint32_t gt = 0u, nc = 0u;
    for (int s = 0; s < steps; ++s) {
        const int i = i0 + 32 * s + lane;
        const uint32_t bin = i < n ? sm.keys[i] >> kBinShift : 0u;
        gt += __popc(__ballot_sync(0xffffffffu, i < n && bin > beta));
        nc += __popc(__ballot_sync(0xffffffffu, i < n && bin == beta));
    }
    uint32_t P;
    uint32_t at = warp_excl_scan(nc, sm.red + kIdxWarps, &P);
    for (int s = 0; s < steps && nc; ++s) {
        const int i = i0 + 32 * s + lane;
        const uint32_t key = i < n ? sm.keys[i] : 0u;
        const bool in = i < n && (key >> kBinShift) == beta;
        const uint32_t m = __ballot_sync(0xffffffffu, in);
        if (in) {
            const uint32_t slot = at + __popc(m & lt);
            sm.u.cand.key[slot] = key;
            sm.u.cand.pos[slot] = static_cast<uint16_t>(i);
        }
        at += __popc(m);
    }
    __syncthreads();
    // 3) exact threshold among the candidates: all keys > thr and the first take_eq == thr
    uint32_t thr = 0u, take_eq = P;
    if (need < P)
        thr = radix_select([&](int c) { return sm.u.cand.key[c]; }, static_cast<int>(P), static_cast<int>(need),
                           sm.rhist, sm.sel + 2, sm.red, &take_eq);
    // 4) selected keys before this warp: above-threshold ones plus the equal ones that fit
    uint32_t ga = gt, eq = 0u;
    for (int s = 0; s < steps && nc; ++s) {
        const int i = i0 + 32 * s + lane;
        const uint32_t key = i < n ? sm.keys[i] : 0u;
        const bool in = i < n && (key >> kBinShift) == beta;
        ga += __popc(__ballot_sync(0xffffffffu, in && key > thr));
        eq += __popc(__ballot_sync(0xffffffffu, in && key == thr));
    }
    uint32_t tot2;
    const uint32_t pre = warp_excl_scan((ga << 16) | eq, sm.red + 2 * kIdxWarps, &tot2);   // counts < 2^16
    uint32_t eq_seen = pre & 0xFFFFu;
    uint32_t pos = (pre >> 16) + min(eq_seen, take_eq);
    // 5) emit in position order
    for (int s = 0; s < steps; ++s) {
        const int i = i0 + 32 * s + lane;
        const uint32_t key = i < n ? sm.keys[i] : 0u;
        const uint32_t bin = key >> kBinShift;
        const bool in = i < n && bin == beta;
        const bool veq = in && key == thr;
        const uint32_t em = __ballot_sync(0xffffffffu, veq);
        const bool take = (i < n && bin > beta) || (in && key > thr) || (veq && eq_seen + __popc(em & lt) < take_eq);
        const uint32_t tm = __ballot_sync(0xffffffffu, take);
        if (take && pos + __popc(tm & lt) < static_cast<uint32_t>(want)) emit(pos + __popc(tm & lt), i);
        pos += __popc(tm);
        eq_seen += __popc(em);
    }
    __syncthreads();
}

// Scores entries c0 .. c0+cn-1 (cn >= 1) of sequence b through an S-stage ring: their order
// keys into keys[0..cn) and their top-11-bit histogram added into hist (zeroed by the caller).
// Returns false (and records CSLD_DEVERR_TIMEOUT) if a copy or an MMA did not complete in
// time.  Called by all 512 threads; allocates and frees NCOLS columns of tensor memory.
// Scoring setup, which reads nothing produced upstream: the ring's barriers and the tensor
// memory (NCOLS columns).  Block-wide; ends with a CTA barrier.
template <int S, uint32_t NCOLS>
__device__ void score_setup(ScoreCtl& ctl) {
    const int tid = threadIdx.x, warp = tid >> 5;
    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&ctl.full[s], 1);
            mbar_init(&ctl.empty[s], 4);          // the 4 warps of the epilogue warpgroup
            mbar_init(&ctl.accf[s], 1);
        }
        mbar_init(&ctl.drain, 1);
        ctl.fail = 0;
        ctl.n_issued = 0;
        ctl.n_mma = 0;
        fence_barrier_init();
    }
    if (warp == kIdxMmaWarp) {
        tmem_alloc(&ctl.tmem_base, NCOLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();   // barriers initialised, tensor memory allocated
    tc_fence_after();
}

// Gives back the tensor memory of score_setup when no chunk is scored.
template <uint32_t NCOLS>
__device__ void score_release(ScoreCtl& ctl) {
    if ((threadIdx.x >> 5) == kIdxMmaWarp) {
        tc_fence_after();
        tmem_dealloc(ctl.tmem_base, NCOLS);
    }
}

// Scores entries c0 .. c0 + cn - 1 of sequence b after score_setup (and gives the tensor
// memory back).  The ring has S tile stages, filled GT tiles at a time: one 1-D bulk copy of
// the GT tiles' key codes (stored pre-swizzled, so the bytes land in the MMA's operand layout)
// and one of their scales, completing on the group's first stage barrier.  Larger copies keep
// the DRAM stream denser than one 8 KB tile per request.
template <int S, int GT, uint32_t NCOLS>
__device__ bool score_run(ScoreCtl& ctl, uint8_t (*codes)[kIdxTile * kIkey], float (*scales)[kIdxTile * 2],
                          uint32_t* keys, uint32_t* hist, uint32_t* stepmax, const uint8_t* ikeys,
                          const float* iscales, int64_t cap, int b, int64_t c0, int cn, const float* q_idx,
                          const float* head_w, int32_t* err) {
    static_assert(S <= kMaxStages, "ring depth");
    static_assert(S % GT == 0 && S / GT >= 2, "the ring holds at least two copy groups");
    static_assert(16 * S + 16 <= static_cast<int>(NCOLS), "accumulator slots and scale factors fit");
    constexpr int kGroups = S / GT;
    constexpr uint32_t kIdxTmemCols = NCOLS, kIdxSfCol = NCOLS - 16;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n_tiles = (cn + kIdxTile - 1) / kIdxTile;
    volatile int32_t* fail = &ctl.fail;
    const uint32_t tmem = ctl.tmem_base;
    const uint8_t* cbase = ikeys + ((size_t)b * cap + (size_t)c0) * kIkey;
    const float* sbase = iscales + ((size_t)b * cap + (size_t)c0) * 2;
    if (warp == kIdxProducerWarp) {
        // --- producer: GT tiles of key codes + their scales per copy group ----------------
        if (lane == 0) {
            int t = 0;
            for (int g = 0; t < n_tiles; ++g) {
                const int s0 = (g % kGroups) * GT;
                if (*fail) break;
                bool free = true;   // the group's stages held tiles t - S .. t - S + GT - 1
                if (g >= kGroups)
                    for (int i = 0; i < GT && free; ++i)
                        free = mbar_wait(&ctl.empty[s0 + i], ((g / kGroups) - 1) & 1);
                if (!free) break;
                const int ne = min(GT * kIdxTile, cn - t * kIdxTile);          // entries in the group
                const uint32_t cb = static_cast<uint32_t>(ne) * kIkey;
                const uint32_t sb = static_cast<uint32_t>((ne + 1) & ~1) * 8u;   // cap is even
                mbar_arrive_expect_tx(&ctl.full[s0], cb + sb);
                bulk_g2s(codes[s0], cbase + (size_t)t * kIdxTile * kIkey, cb, &ctl.full[s0]);
                bulk_g2s(scales[s0], sbase + (size_t)t * kIdxTile * 2, sb, &ctl.full[s0]);
                t = min(n_tiles, t + GT);
            }
            ctl.n_issued = t;
            if (t < n_tiles) *fail = 1;
        }
    } else {
        // --- query operand: FP4 codes in the MMA's B layout (8 rows x 32 bytes, 32-byte
        // swizzle), prepared while the producer already streams.  Row n is head n & 3 over
        // group n >> 2; the row's other 32-element group is zero, so every output column is one
        // exact group dot.  Thread t writes bytes 4j..4j+3 of row n.
        if (tid < 64) {
            const int n = tid >> 3, j = tid & 7, h = n & 3, grp = n >> 2;
            const float4* qv = reinterpret_cast<const float4*>(q_idx + ((size_t)b * kIdxHeads + h) * kIdxDim + 32 * grp);
            float amax = 0.f;
            float4 lo = make_float4(0.f, 0.f, 0.f, 0.f), hi = lo;   // dims 8(j&3)..8(j&3)+7 of the group
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float4 t = __ldg(qv + i);
                amax = fmaxf(fmaxf(fmaxf(amax, fabsf(t.x)), fmaxf(fabsf(t.y), fabsf(t.z))), fabsf(t.w));
                if (i == 2 * (j & 3)) lo = t;
                if (i == 2 * (j & 3) + 1) hi = t;
            }
            const float sg = fp4_group_scale(amax);
            const float inv = 1.0f / sg;   // exact: a power of two
            uint32_t word = 0u;
            if ((j >> 2) == grp) {         // dims 8j..8j+7 = group dims 8(j&3)..8(j&3)+7
                const float x[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
                for (int i = 0; i < 8; ++i) word |= e2m1_code(x[i] * inv) << (4 * i);
            }
            const int half = (j >> 2) ^ ((n >> 2) & 1);
            *reinterpret_cast<uint32_t*>(ctl.bq + n * kIkey + half * 16 + (j & 3) * 4) = word;
            if (j == 0) ctl.qscale[grp * 4 + h] = sg;
            fence_proxy_async_smem();
        }
        if (warp < 4) {   // unit block-scale factors (UE8M0 0x7F = 2^0) for A and B, every lane
            tmem_st_32x32b_x8_fill(tmem + ((32u * warp) << 16) + kIdxSfCol, 0x7F7F7F7Fu);
            tmem_st_32x32b_x8_fill(tmem + ((32u * warp) << 16) + kIdxSfCol + 8, 0x7F7F7F7Fu);
            tmem_st_wait();
        }
        tc_fence_before();
        named_barrier(1, kIdxThreads - 32);   // every warp but the producer
        tc_fence_after();
        if (warp == kIdxMmaWarp) {
            // --- MMA issuer: two 128-row block-scaled FP4 MMAs per tile into accumulator slot s
            if (lane == 0) {
                const uint64_t bdesc = smem_desc_kmajor_sw32(ctl.bq);
                const uint32_t sfa = tmem + kIdxSfCol, sfb = tmem + kIdxSfCol + 8;
                int t = 0;
                for (; t < n_tiles; ++t) {
                    const int s = t % S;
                    // a copy group lands as a whole on the barrier of its first stage
                    if (*fail || (t % GT == 0 && !mbar_wait(&ctl.full[s], ((t / GT) / kGroups) & 1))) break;
                    tc_fence_after();
                    const uint32_t d = tmem + 16u * static_cast<uint32_t>(s);
                    umma_mxf4(d, smem_desc_kmajor_sw32(codes[s]), bdesc, kIdxIdesc, sfa, sfb, 0u);
                    umma_mxf4(d + 8u, smem_desc_kmajor_sw32(codes[s] + 128 * kIkey), bdesc, kIdxIdesc,
                              sfa, sfb, 0u);
                    umma_commit(&ctl.accf[s]);
                }
                ctl.n_mma = t;
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
            for (int i = 0; i < 8; ++i) qsc[i] = ctl.qscale[i];
            const float w0 = head_w[b * kIdxHeads + 0], w1 = head_w[b * kIdxHeads + 1];
            const float w2 = head_w[b * kIdxHeads + 2], w3 = head_w[b * kIdxHeads + 3];
            for (int t = wg; t < n_tiles; t += kIdxEpiGroups) {
                const int s = t % S;
                const bool landed = !*fail && mbar_wait(&ctl.accf[s], (t / S) & 1);
                if (!__all_sync(0xffffffffu, landed)) {
                    if (lane == 0) *fail = 1;
                    break;
                }
                tc_fence_after();
                uint32_t r[16];
                tmem_ld_32x32b_x16(lane_addr + 16u * static_cast<uint32_t>(s), r);
                tmem_ld_wait();
                const float2* ss = reinterpret_cast<const float2*>(scales[s]);
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
                    const uint32_t key = score_key(sc);
                    if (li < cn) keys[li] = key;
                    if (li < cn) atomicAdd(&hist[key >> kBinShift], 1u);   // plain: scores spread over bins
                    if (stepmax != nullptr) {   // the warp's 32 entries are one aligned step
                        const uint32_t mx = __reduce_max_sync(0xffffffffu, li < cn ? key : 0u);
                        if (lane == 0) stepmax[li >> 5] = mx;
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&ctl.empty[s]);   // stage s and accumulator slot s free
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    const bool ok = (ctl.fail == 0);
    if (!ok) {
        // A copy or an MMA did not complete in time: record it, let the copies in flight
        // land and the MMAs in flight finish (bounded waits) before the shared and tensor
        // memory are reused.
        if (warp == kIdxMmaWarp && lane == 0) {
            dev_error(err, CSLD_DEVERR_TIMEOUT);
            for (int t = (ctl.n_mma + GT - 1) / GT * GT; t < ctl.n_issued; t += GT)
                (void)mbar_wait(&ctl.full[t % S], ((t / GT) / kGroups) & 1);
            umma_commit(&ctl.drain);
            (void)mbar_wait(&ctl.drain, 0);
        }
        __syncthreads();
    }
    if (warp == kIdxMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kIdxTmemCols);
    }
    return ok;
}

template <int S, int GT, uint32_t NCOLS>
__device__ bool score_chunk(ScoreCtl& ctl, uint8_t (*codes)[kIdxTile * kIkey], float (*scales)[kIdxTile * 2],
                            uint32_t* keys, uint32_t* hist, const uint8_t* ikeys, const float* iscales,
                            int64_t cap, int b, int64_t c0, int cn, const float* q_idx, const float* head_w,
                            int32_t* err) {
    score_setup<S, NCOLS>(ctl);
    return score_run<S, GT, NCOLS>(ctl, codes, scales, keys, hist, nullptr, ikeys, iscales, cap, b, c0, cn, q_idx, head_w,
                                   err);
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
// The merge-tree kernel.
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kIdxThreads, 2) indexer_topk_kernel(
    const uint8_t* __restrict__ ikeys, const float* __restrict__ iscales, int64_t cap,
    const int32_t* __restrict__ seq_len, int ratio, const float* __restrict__ q_idx,
    const float* __restrict__ head_w, int chunk, int kc, int k, IdxTree tree,
    int32_t* __restrict__ topk_out, int32_t* err) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    IdxSmem& sm = *reinterpret_cast<IdxSmem*>(
        smem_raw + ((kIdxSmemAlign - (smem_u32(smem_raw) & (kIdxSmemAlign - 1))) & (kIdxSmemAlign - 1)));
    const int tid = threadIdx.x;
    const int b = blockIdx.y, ch = blockIdx.x;

    int64_t n_b = seq_len[b];
    n_b = n_b < 0 ? 0 : n_b / ratio;
    if (n_b > cap) n_b = cap;
    const int64_t c0 = (int64_t)ch * chunk;
    const int cn = static_cast<int>(max64(0, min64(chunk, n_b - c0)));

    for (int i = tid; i < kBins; i += blockDim.x) sm.hist[i] = 0u;
    bool chunk_ok = true;
    if (cn > 0)
        chunk_ok = score_chunk<kIdxStages, 1, 128>(sm.ctl, sm.u.pipe.codes, sm.u.pipe.scales, sm.keys, sm.hist, ikeys, iscales,
                                           cap, b, c0, cn, q_idx, head_w, err);
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
                kv[u] = 0u;
                if (c < children && i < sm.offs[c + 1] - sm.offs[c]) {
                    kv[u] = __ldcg(tree.keys[level] + child0 + flat);
                    dst[u] = sm.offs[c] + i;
                }
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                if (dst[u] >= 0) sm.keys[dst[u]] = kv[u];
                hist_add(sm.hist, kv[u] >> kBinShift, dst[u] >= 0);
            }
        }
        child_idx = reinterpret_cast<const uint32_t*>(tree.idx[level] + child0);
        n = sm.offs[children];
        __syncthreads();
        ++level;
        run = parent;
    }
}

// ------------------------------------------------------------------------------------------
// The cooperative kernel: one exact radix select per sequence across its CTAs.
// ------------------------------------------------------------------------------------------
struct CoopWs {
    uint32_t* hist;    // [B][2][kCoopSeqWords]: level 1 (2048 bins), level 2 (2048), level 3 (1024)
    uint32_t* sync;    // [B][64]: words 0-1 barrier arrivals, 2-3 list length (one per set), 4 epoch
    uint32_t* counts;  // [B][2][units][2]: keys above the threshold, keys equal to it
    uint64_t* lslot;   // [B][2][kListMax]: candidate list, (range + 1) << 32 | key; 0 = not written
};

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Barrier of the CTAs of one sequence: arrival counter *ctr reaches `target`.  The spin is
// bounded (about half a second); on time-out the device error word gets CSLD_DEVERR_TIMEOUT
// and false is returned to every thread of the CTA.  The CTA barrier orders every thread's
// global writes before thread 0's arrival, a release add (release is cumulative), and thread
// 0's acquire load of the count orders the other CTAs' writes before everything the CTA does
// after the closing barrier, as in a grid-wide sync.
__device__ bool seq_barrier(uint32_t* ctr, uint32_t target, int32_t* fail_flag, int32_t* err) {
    __syncthreads();
    if (threadIdx.x == 0) {
        // a release add: the CTA's writes before the barrier above are visible to whoever
        // acquires the count (no separate fence, and no wait for the add's return value)
        asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(ctr) : "memory");
        bool ok = false;
        for (uint32_t i = 0; i < (1u << 22); ++i) {
            if (ld_acquire_u32(ctr) >= target) {
                ok = true;
                break;
            }
            if (i >= 64) __nanosleep(32);
        }
        if (!ok) {
            dev_error(err, CSLD_DEVERR_TIMEOUT);
            *fail_flag = 1;
        }
    }
    __syncthreads();
    return *reinterpret_cast<volatile int32_t*>(fail_flag) == 0;
}

__device__ __forceinline__ void st_relaxed_u32(uint32_t* p, uint32_t v) {
    asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" :: "l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void st_relaxed_u64(uint64_t* p, uint64_t v) {
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" :: "l"(p), "l"(v) : "memory");
}
// A word another CTA of the sequence writes once (from zero) during this call: polled until it
// is non-zero, about a second at most; 0 if it never was.
__device__ __forceinline__ uint32_t poll_nonzero_u32(const uint32_t* p) {
    for (uint32_t i = 0; i < (1u << 22); ++i) {
        uint32_t v;
        asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
        if (v != 0u) return v;
        if (i >= 64) __nanosleep(32);
    }
    return 0u;
}
__device__ __forceinline__ uint64_t poll_nonzero_u64(const uint64_t* p) {
    for (uint32_t i = 0; i < (1u << 22); ++i) {
        uint64_t v;
        asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
        if (v != 0ull) return v;
        if (i >= 64) __nanosleep(32);
    }
    return 0ull;
}

// From a global histogram g of nbins bins (2048 or 1024), the bin holding the want-th largest
// key and how many keys are wanted inside it (*need).  Block-wide; g read through L2.
__device__ void find_bin_global(const uint32_t* g, int nbins, uint32_t want, uint32_t* red, uint32_t* sel,
                                uint32_t* bin, uint32_t* need, uint32_t* count = nullptr) {
    const int tid = threadIdx.x, lane = tid & 31;
    const int per = nbins / kIdxThreads;     // 4 or 2 bins per thread, from the top
    uint32_t c[4] = {0u, 0u, 0u, 0u}, tot = 0u;
    for (int q = 0; q < per; ++q) {
        c[q] = __ldcg(g + nbins - 1 - per * tid - q);
        tot += c[q];
    }
    uint32_t incl = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (tid == 0) {
        sel[0] = 0u;
        sel[1] = 0u;
        sel[2] = 0u;
    }
    uint32_t all;
    const uint32_t wb = warp_excl_scan(__shfl_sync(0xffffffffu, incl, 31), red, &all);
    const uint32_t excl = wb + incl - tot;
    if (excl < want && excl + tot >= want) {
        uint32_t run = excl;
        for (int q = 0; q < per; ++q) {
            if (run + c[q] >= want) {
                sel[0] = static_cast<uint32_t>(nbins - 1 - per * tid - q);
                sel[1] = want - run;
                sel[2] = c[q];
                break;
            }
            run += c[q];
        }
    }
    __syncthreads();
    *bin = sel[0];
    *need = sel[1];
    if (count != nullptr) *count = sel[2];
    __syncthreads();
}

// Level 1 without a barrier: the sequence's global histogram g (kBins bins) is complete once its
// bins add up to `total`, the number of keys its ranges scored (bins only grow, so a read whose
// sum is the total holds every bin's final count).  Re-read until it is (bounded: about half a
// second, then CSLD_DEVERR_TIMEOUT and false in every thread); then, as find_bin_global, the bin
// holding the want-th largest key, the keys wanted inside it and the bin's count.
__device__ bool find_bin_complete(const uint32_t* g, uint32_t total, uint32_t want, uint32_t* red, uint32_t* sel,
                                  uint32_t* bin, uint32_t* need, uint32_t* count, int32_t* err) {
    const int tid = threadIdx.x, lane = tid & 31;
    constexpr int per = kBins / kIdxThreads;
    uint32_t c[per], tot = 0u, incl = 0u, wb = 0u, all = 0u;
    bool ok = false;
    for (uint32_t it = 0; it < (1u << 20); ++it) {
        tot = 0u;
#pragma unroll
        for (int q = 0; q < per; ++q) {
            asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(c[q]) : "l"(g + kBins - 1 - per * tid - q) : "memory");
            tot += c[q];
        }
        incl = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        wb = warp_excl_scan(__shfl_sync(0xffffffffu, incl, 31), red, &all);
        __syncthreads();   // red is written again by the next read
        if (all == total) {
            ok = true;
            break;
        }
        if (it >= 16) __nanosleep(64);
    }
    if (!ok) {
        if (tid == 0) dev_error(err, CSLD_DEVERR_TIMEOUT);
        return false;
    }
    if (tid == 0) {
        sel[0] = 0u;
        sel[1] = 0u;
        sel[2] = 0u;
    }
    __syncthreads();
    const uint32_t excl = wb + incl - tot;
    if (excl < want && excl + tot >= want) {
        uint32_t run = excl;
        for (int q = 0; q < per; ++q) {
            if (run + c[q] >= want) {
                sel[0] = static_cast<uint32_t>(kBins - 1 - per * tid - q);
                sel[1] = want - run;
                sel[2] = c[q];
                break;
            }
            run += c[q];
        }
    }
    __syncthreads();
    *bin = sel[0];
    *need = sel[1];
    *count = sel[2];
    __syncthreads();
    return true;
}

__global__ void __launch_bounds__(kIdxThreads, 1) indexer_topk_coop_kernel(
    const uint8_t* __restrict__ ikeys, const float* __restrict__ iscales, int64_t cap,
    const int32_t* __restrict__ seq_len, int ratio, const float* __restrict__ q_idx,
    const float* __restrict__ head_w, int chunk, int units, int k, CoopWs ws,
    int32_t* __restrict__ topk_out, int32_t* err, uint32_t barrier_extra) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    CoopSmem& sm = *reinterpret_cast<CoopSmem*>(
        smem_raw + ((kIdxSmemAlign - (smem_u32(smem_raw) & (kIdxSmemAlign - 1))) & (kIdxSmemAlign - 1)));
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t lt = (1u << lane) - 1u;
    const int b = blockIdx.y, u = blockIdx.x;

    for (int i = tid; i < kBins; i += blockDim.x) {
        sm.hist[i] = 0u;
        sm.hist2[i] = 0u;
    }
    for (int i = tid; i < 1024; i += blockDim.x) sm.hist3[i] = 0u;
    if (tid == 0) sm.fail = 0;
    score_setup<kCoopStages, 256>(sm.ctl);

    int64_t n_b = seq_len[b];
    n_b = n_b < 0 ? 0 : n_b / ratio;
    if (n_b > cap) n_b = cap;
    // this CTA's range: an even share of the sequence's visible tiles (the plan's chunk, sized
    // from cap, bounds it), so the last range is not left short
    const int64_t tiles_b = (n_b + kIdxTile - 1) / kIdxTile;
    const int64_t c0 = tiles_b * u / units * kIdxTile;
    const int cn = static_cast<int>(max64(0, min64(min64(tiles_b * (u + 1) / units * kIdxTile, n_b) - c0, chunk)));
    int32_t* out = topk_out + (size_t)b * k;

    if (n_b <= k) {
        // every visible entry is selected: no scores needed, and no barrier (the whole
        // sequence takes this branch); entry i goes to position i, the rest is -1
        score_release<256>(sm.ctl);
        for (int i = tid; i < cn; i += blockDim.x) out[c0 + i] = static_cast<int32_t>(c0 + i);
        if (u == 0)
            for (int64_t i = n_b + tid; i < k; i += blockDim.x) out[i] = -1;
        return;
    }
    const uint32_t want = static_cast<uint32_t>(k);
    // Two sets of selection state (histograms, barrier counter, list length, candidate list,
    // per-range counts) per sequence; the epoch (calls completed on this sequence) picks this
    // call's set.  The other set belonged to the previous call, which has finished: every CTA
    // clears its share of it here for the next call, so nothing has to be reset at the end of
    // this one.  Every CTA reads the epoch before it adds to the level-1 histogram, and range 0
    // advances it at its end, after it has seen the complete histogram.
    uint32_t* sq = ws.sync + (size_t)b * 64;
    const uint32_t par = __ldcg(sq + 4) & 1u;
    uint32_t* g1 = ws.hist + ((size_t)b * 2 + par) * kCoopSeqWords;
    uint32_t* g2 = g1 + kBins;
    uint32_t* g3 = g2 + kBins;
    uint32_t* bar = sq + par;
    uint32_t* cnt = ws.counts + ((size_t)b * 2 + par) * units * 2;
    uint32_t* lcount = sq + 2 + par;
    uint64_t* lslot = ws.lslot + ((size_t)b * 2 + par) * kListMax;
    {
        uint32_t* other = ws.hist + ((size_t)b * 2 + (par ^ 1u)) * kCoopSeqWords;
        int lo = kCoopSeqWords * u / units, hi = kCoopSeqWords * (u + 1) / units;
        for (int i = lo + tid; i < hi; i += blockDim.x) other[i] = 0u;
        uint64_t* olist = ws.lslot + ((size_t)b * 2 + (par ^ 1u)) * kListMax;
        lo = kListMax * u / units;
        hi = kListMax * (u + 1) / units;
        for (int i = lo + tid; i < hi; i += blockDim.x) olist[i] = 0ull;
        if (u == 0) {
            uint32_t* ocnt = ws.counts + ((size_t)b * 2 + (par ^ 1u)) * units * 2;
            for (int i = tid; i < 2 * units; i += blockDim.x) ocnt[i] = 0u;
            if (tid == 0) {
                sq[par ^ 1u] = 0u;
                sq[2 + (par ^ 1u)] = 0u;
            }
        }
    }
    const uint32_t nu = static_cast<uint32_t>(units);

    bool ok = true;
    if (cn > 0)
        ok = score_run<kCoopStages, kCoopGroup, 256>(sm.ctl, sm.codes, sm.scales, sm.keys, sm.hist, sm.stepmax, ikeys,
                                                     iscales, cap, b,
                                                     c0, cn,
                                         q_idx, head_w, err);
    else
        score_release<256>(sm.ctl);
    __syncthreads();
    // --- level 1: bits 31..21.  No barrier: every CTA re-reads the sequence's histogram until it
    //     holds all n_b keys (the ranges partition the visible entries).  A range whose scoring
    //     timed out adds its key count to bin 0, so the others still get past this point (the
    //     error word already says the selection is not to be trusted). ---------------------------
    if (ok) {
        for (int i = tid; i < kBins; i += blockDim.x) {
            const uint32_t c = sm.hist[i];
            if (c) atomicAdd(g1 + i, c);
        }
    } else if (tid == 0 && cn > 0) {
        atomicAdd(g1, static_cast<uint32_t>(cn));
    }
    uint32_t beta1, need1, cnt1;
    if (!find_bin_complete(g1, static_cast<uint32_t>(n_b) + barrier_extra, want, sm.red, sm.sel, &beta1, &need1,
                           &cnt1, err))
        return;
    // --- candidates: one pass over the range.  Each warp counts its keys above bin beta1 and
    //     copies the keys inside it to its own candidate region (the copy ring is idle now).
    //     When the sequence's bin beta1 is small, the candidates of all its ranges go to one
    //     global list that every CTA then resolves on its own (no barrier); otherwise two more
    //     histogram levels run (bits 20..10, then 9..0) and the ranges exchange their counts
    //     (three barriers).  The choice is the same in every CTA of the sequence. --------
    const bool fast = cnt1 <= static_cast<uint32_t>(kListMax) && units <= 255;
    constexpr int kSeg = kCoopMaxRange / kIdxWarps;    // warp w owns positions 1024w .. 1024w+1023
    uint32_t* cand = reinterpret_cast<uint32_t*>(&sm.codes[0][0]) + warp * kSeg;
    const int i0 = warp * kSeg;
    const int steps = max(0, min(kSeg, cn - i0) + 31) >> 5;
    uint32_t gt = 0u, nc = 0u;
    // 32-key steps of this warp's segment holding a key of bin >= beta1, from the step maxima
    // kept while scoring (steps <= 32); only they can hold a key above or inside bin beta1
    const uint32_t cmask = __ballot_sync(0xffffffffu, lane < steps && sm.stepmax[(i0 >> 5) + lane] >= (beta1 << kBinShift));
    for (uint32_t mk = cmask; mk != 0u; mk &= mk - 1u) {
        const int s = __ffs(mk) - 1;
        const int i = i0 + 32 * s + lane;
        const uint32_t key = i < cn ? sm.keys[i] : 0u;
        const uint32_t bin = key >> kBinShift;
        const uint32_t ma = __ballot_sync(0xffffffffu, i < cn && bin > beta1);
        gt += __popc(ma);
        const bool in = i < cn && bin == beta1;
        const uint32_t m = __ballot_sync(0xffffffffu, in);
        if (in) {
            cand[nc + __popc(m & lt)] = key;
            if (!fast) {   // level-2 histogram: bits 20..10
                const uint32_t sub = (key >> 10) & (kBins - 1);
                const uint32_t same = __match_any_sync(m, sub);   // lanes sharing a bin: one atomic
                if (lane == __ffs(same) - 1) atomicAdd(&sm.hist2[sub], static_cast<uint32_t>(__popc(same)));
            }
        }
        nc += __popc(m);
    }
    const int csteps = static_cast<int>((nc + 31) >> 5);
    uint32_t thr, take_eq, A, E;
    if (fast) {
        // this range's candidates -> the sequence's list; its keys above bin beta1 -> counts
        uint32_t nc_all, gt_all;
        const uint32_t woff = warp_excl_scan(nc, sm.red + kIdxWarps, &nc_all);
        (void)warp_excl_scan(gt, sm.red + 2 * kIdxWarps, &gt_all);
        if (tid == 0) {
            sm.sel[2] = atomicAdd(lcount, nc_all);
            st_relaxed_u32(cnt + 2 * u, gt_all + 1u);   // + 1: zero means not written yet
        }
        __syncthreads();
        const uint32_t lbase = sm.sel[2] + woff;
        for (int j = lane; j < static_cast<int>(nc); j += 32) {
            const uint32_t at = lbase + static_cast<uint32_t>(j);
            if (at < static_cast<uint32_t>(kListMax))
                st_relaxed_u64(lslot + at, (static_cast<uint64_t>(u + 1) << 32) | cand[j]);
        }
        // No second barrier: the list holds exactly cnt1 entries (the global histogram's count
        // of bin beta1), so every CTA reads slots 0 .. cnt1 - 1, each as soon as it is written,
        // into the ring's last 32 KB (keys) and hist2 (range ids), and finds the exact
        // threshold among them.  Every wait is bounded.
        const int P = static_cast<int>(min(cnt1, static_cast<uint32_t>(kListMax)));
        uint32_t* lk = reinterpret_cast<uint32_t*>(&sm.codes[0][0]) + kCoopMaxRange;
        uint8_t* lu = reinterpret_cast<uint8_t*>(sm.hist2);
        uint32_t a_loc = 0u, e_loc = 0u;
        bool waited = true;
        for (int v = tid; v < u && waited; v += blockDim.x) {
            const uint32_t c = poll_nonzero_u32(cnt + 2 * v);
            waited = c != 0u;
            a_loc += c - 1u;
        }
        for (int i0 = tid; i0 < P && waited; i0 += 4 * kIdxThreads) {
            uint64_t w[4];   // four slots in flight; re-read only those not written yet
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int i = i0 + q * kIdxThreads;
                w[q] = 1ull;
                if (i < P) asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(w[q]) : "l"(lslot + i) : "memory");
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int i = i0 + q * kIdxThreads;
                if (i < P) {
                    if (w[q] == 0ull) w[q] = poll_nonzero_u64(lslot + i);
                    waited = waited && w[q] != 0ull;
                    lk[i] = static_cast<uint32_t>(w[q]);
                    lu[i] = static_cast<uint8_t>((w[q] >> 32) - 1u);
                }
            }
        }
        if (tid < 256) sm.hist[tid] = 0u;
        if (__syncthreads_or(!waited)) {
            if (tid == 0) dev_error(err, CSLD_DEVERR_TIMEOUT);
            return;
        }
        // when the whole of bin beta1 is wanted, its lowest key is the threshold (every key
        // equal to it taken): keys of lower bins, which the emit pass also visits, stay below it
        thr = beta1 << kBinShift;
        take_eq = static_cast<uint32_t>(P);
        if (static_cast<int>(need1) < P)
            thr = list_select(lk, P, need1, beta1 << kBinShift, sm.hist, sm.sel + 2, &take_eq);
        // selected before this range: the earlier ranges' keys above bin beta1 (a_loc, loaded
        // above), and their candidates above / equal to the threshold
        for (int i = tid; i < P; i += blockDim.x)
            if (lu[i] < u) {
                a_loc += lk[i] > thr;
                e_loc += lk[i] == thr;
            }
        block_sum2(a_loc, e_loc, sm.red + kIdxWarps, &A, &E);
    } else {
        __syncthreads();
        for (int i = tid; i < kBins; i += blockDim.x) {
            const uint32_t c = sm.hist2[i];
            if (c) atomicAdd(g2 + i, c);
        }
        if (!seq_barrier(bar, 1 * nu + barrier_extra, &sm.fail, err)) return;
        uint32_t beta2, need2;
        find_bin_global(g2, kBins, need1, sm.red, sm.sel, &beta2, &need2);
        const uint32_t top22 = (beta1 << 11) | beta2;
        // level 3: bits 9..0 of the candidates whose top 22 bits are (beta1, beta2)
        for (int s = 0; s < csteps; ++s) {
            const int j = 32 * s + lane;
            const uint32_t key = j < static_cast<int>(nc) ? cand[j] : 0u;
            const bool in = j < static_cast<int>(nc) && (key >> 10) == top22;
            const uint32_t m = __ballot_sync(0xffffffffu, in);
            if (in) {
                const uint32_t low = key & 1023u;
                const uint32_t same = __match_any_sync(m, low);
                if (lane == __ffs(same) - 1) atomicAdd(&sm.hist3[low], static_cast<uint32_t>(__popc(same)));
            }
        }
        __syncthreads();
        for (int i = tid; i < 1024; i += blockDim.x) {
            const uint32_t c = sm.hist3[i];
            if (c) atomicAdd(g3 + i, c);
        }
        if (!seq_barrier(bar, 2 * nu + barrier_extra, &sm.fail, err)) return;
        uint32_t beta3;
        find_bin_global(g3, 1024, need2, sm.red, sm.sel, &beta3, &take_eq);
        thr = (top22 << 10) | beta3;
        // this range's counts, then the counts of the ranges before it
        uint32_t above = 0u, equal = 0u;
        for (int s = 0; s < csteps; ++s) {
            const int j = 32 * s + lane;
            const uint32_t key = j < static_cast<int>(nc) ? cand[j] : 0u;
            above += j < static_cast<int>(nc) && key > thr;
            equal += j < static_cast<int>(nc) && key == thr;
        }
        above = gt + __reduce_add_sync(0xffffffffu, above);
        equal = __reduce_add_sync(0xffffffffu, equal);
        uint32_t tot;
        (void)warp_excl_scan((above << 16) | equal, sm.red + kIdxWarps, &tot);   // counts <= 2^14
        if (tid == 0) {
            cnt[2 * u] = tot >> 16;
            cnt[2 * u + 1] = tot & 0xFFFFu;
        }
        if (!seq_barrier(bar, 3 * nu + barrier_extra, &sm.fail, err)) return;
        uint32_t a_loc = 0u, e_loc = 0u;
        for (int v = tid; v < u; v += blockDim.x) {
            a_loc += __ldcg(cnt + 2 * v);
            e_loc += __ldcg(cnt + 2 * v + 1);
        }
        block_sum2(a_loc, e_loc, sm.red + kIdxWarps, &A, &E);
    }
    // this warp's selected keys: above bin beta1, and candidates above / equal to thr
    uint32_t above = 0u, equal = 0u;
    for (int s = 0; s < csteps; ++s) {
        const int j = 32 * s + lane;
        const uint32_t key = j < static_cast<int>(nc) ? cand[j] : 0u;
        above += j < static_cast<int>(nc) && key > thr;
        equal += j < static_cast<int>(nc) && key == thr;
    }
    above = gt + __reduce_add_sync(0xffffffffu, above);
    equal = __reduce_add_sync(0xffffffffu, equal);
    uint32_t tot;
    const uint32_t pre = warp_excl_scan((above << 16) | equal, sm.red + kIdxWarps, &tot);   // counts <= 2^14
    // --- emit this range's selected entries in index order ------------------------------------
    uint32_t eq_seen = E + (pre & 0xFFFFu);
    uint32_t pos = A + (pre >> 16) + min(eq_seen, take_eq);
    // only steps with a key of bin >= beta1 can hold a selected key (the threshold lies in bin
    // beta1), so the others are skipped
    for (uint32_t mk = cmask; mk != 0u; mk &= mk - 1u) {
        const int s = __ffs(mk) - 1;
        const int i = i0 + 32 * s + lane;
        const uint32_t key = i < cn ? sm.keys[i] : 0u;
        const bool veq = i < cn && key == thr;
        const uint32_t em = __ballot_sync(0xffffffffu, veq);
        const bool take = (i < cn && key > thr) || (veq && eq_seen + __popc(em & lt) < take_eq);
        const uint32_t tm = __ballot_sync(0xffffffffu, take);
        const uint32_t at = pos + __popc(tm & lt);
        // the counts add up to exactly k when every range scored; after a timed-out range the
        // positions are not trusted
        if (take && at < want) out[at] = static_cast<int32_t>(c0 + i);
        pos += __popc(tm);
        eq_seen += __popc(em);
    }
    // --- this call is over for the sequence: the next one takes the other state set ------------
    if (u == 0 && tid == 0) atomicAdd(sq + 4, 1u);
}

// Test hook (csld_test_set_barrier_extra): added to the key total the level-1 histogram must
// reach and to every cross-CTA barrier target of the cooperative kernel, so that a test can make
// its bounded waits run out.  0 in normal use.
std::atomic<int> g_test_barrier_extra{0};

// Resident CTAs of the cooperative kernel on the current device (0 if it cannot run), found
// once per device.
static int coop_slots(int num_sms) {
    constexpr int kMaxDev = 64;
    static std::mutex mu;
    static int per_sm[kMaxDev];
    static bool known[kMaxDev] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) {
        (void)cudaGetLastError();
        return 0;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (!known[dev]) {
        const size_t smem = sizeof(CoopSmem) + kIdxSmemAlign;
        int n = 0;
        if (set_smem_once(indexer_topk_coop_kernel, smem) == cudaSuccess &&
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, indexer_topk_coop_kernel, kIdxThreads, smem) ==
                cudaSuccess)
            per_sm[dev] = n;
        else
            per_sm[dev] = 0;
        (void)cudaGetLastError();
        known[dev] = true;
    }
    return per_sm[dev] * num_sms;
}

static size_t coop_layout(int B, int units, uint8_t* base, CoopWs* ws) {
    const size_t h = up256((size_t)B * 2 * kCoopSeqWords * 4), s = up256((size_t)B * 64 * 4),
                 c = up256((size_t)B * 2 * units * 2 * 4), lk = up256((size_t)B * 2 * kListMax * 8);
    if (ws) {
        ws->hist = reinterpret_cast<uint32_t*>(base);
        ws->sync = reinterpret_cast<uint32_t*>(base + h);
        ws->counts = reinterpret_cast<uint32_t*>(base + h + s);
        ws->lslot = reinterpret_cast<uint64_t*>(base + h + s + c);
    }
    return h + s + c + lk;
}

IndexerPlan indexer_plan(int B, int64_t cap, int k, int num_sms) {
    IndexerPlan p{};
    // Cooperative path: every sequence split into `units` ranges of at most kCoopMaxRange
    // entries (a multiple of the tile), all B * units CTAs resident at once (one per SM: the
    // occupancy the runtime grants a kernel that allocates tensor memory).
    const int slots = coop_slots(num_sms);
    if (slots > 0) {
        const int64_t per_seq = max64(1, slots / B);
        int64_t chunk = (cap + per_seq - 1) / per_seq;
        chunk = max64(kIdxTile, (chunk + kIdxTile - 1) / kIdxTile * kIdxTile);
        const int64_t units = (cap + chunk - 1) / chunk;
        if (chunk <= kCoopMaxRange && (int64_t)B * units <= slots) {
            p.coop = true;
            p.chunk = static_cast<int>(chunk);
            p.n_chunks = static_cast<int>(units);
            p.kc = k < chunk ? k : static_cast<int>(chunk);
            p.group = 0;
            p.levels_ok = true;
            p.ws_bytes = coop_layout(B, p.n_chunks, nullptr, nullptr);
            return p;
        }
    }
    // Merge-tree path: chunks of all sequences spread over the SMs (2 CTAs each) as evenly as
    // possible, a multiple of the tile between 1024 and kIdxMaxChunk entries.
    const int64_t per_seq = max64(1, (2LL * num_sms) / B);
    int64_t chunk = (cap + per_seq - 1) / per_seq;
    chunk = (chunk + kIdxTile - 1) / kIdxTile * kIdxTile;
    chunk = max64(1024, min64(kIdxMaxChunk, chunk));
    p.chunk = static_cast<int>(chunk);
    const int64_t nc = (cap + chunk - 1) / chunk;
    p.n_chunks = static_cast<int>(nc < 1 ? 1 : nc);
    p.kc = k < chunk ? k : static_cast<int>(chunk);
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

bool make_tensor_map_2d_u8(CUtensorMap* map, const void* base, uint64_t row_bytes, uint64_t rows, uint32_t box_x,
                           uint32_t box_y) {
    PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
    if (encode == nullptr) return false;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(row_bytes), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_bytes)};
    const cuuint32_t box[2] = {box_x, box_y};
    const cuuint32_t estr[2] = {1u, 1u};
    return encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_indexer(const uint8_t* ikeys, const float* iscales, int64_t cap,
                           const int32_t* seq_len, int ratio, const float* q_idx,
                           const float* head_w, int B, int k, int32_t* topk_out, void* ws,
                           const IndexerPlan& plan, int32_t* err, cudaStream_t stream) {
    if (plan.coop) {
        CoopWs cws;
        coop_layout(B, plan.n_chunks, static_cast<uint8_t*>(ws), &cws);
        const size_t smem = sizeof(CoopSmem) + kIdxSmemAlign;
        cudaError_t e = set_smem_once(indexer_topk_coop_kernel, smem);
        if (e != cudaSuccess) return e;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(plan.n_chunks, B);
        cfg.blockDim = dim3(kIdxThreads);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeCooperative;   // all CTAs resident: the barriers can complete
        attr[0].val.cooperative = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, indexer_topk_coop_kernel, ikeys, iscales, cap, seq_len, ratio, q_idx, head_w,
                               plan.chunk, plan.n_chunks, k, cws, topk_out, err,
                               static_cast<uint32_t>(g_test_barrier_extra.load()));
        if (e != cudaSuccess) return e;
        return cudaGetLastError();
    }
    size_t bytes = 0;
    IdxTree tree = tree_layout(B, plan.n_chunks, plan.kc, k, plan.group, static_cast<uint8_t*>(ws), &bytes);
    const size_t smem = sizeof(IdxSmem) + kIdxSmemAlign;
    cudaError_t e = set_smem_once(indexer_topk_kernel, smem);
    if (e != cudaSuccess) return e;
    dim3 grid(plan.n_chunks, B);
    indexer_topk_kernel<<<grid, kIdxThreads, smem, stream>>>(ikeys, iscales, cap, seq_len, ratio,
                                                             q_idx, head_w, plan.chunk, plan.kc, k,
                                                             tree, topk_out, err);
    return cudaGetLastError();
}

}  // namespace csld
