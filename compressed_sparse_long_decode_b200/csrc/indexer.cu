// Lightning indexer + exact top-k.
//
// Source: "DeepSeek-V4: a million-token context that agents can actually use" -- CSA paragraph
// (the lightning indexer, an FP4 ReLU-scored multi-head dot product, picks the top-k
// compressed blocks for each query) and Figure 3 caption; velog.io paper review, "core
// technique 1: CSA" (the indexer scores which compressed entries the query should read).
//
// Score of entry s for one query (4 heads, 64 dims, one key per entry shared by the heads):
//   e_s = sum_h w_h * ReLU(q_h . k_s), q and k both FP4 (E2M1 codes, power-of-two scale / 32).
// The two 32-element group dots of every (entry, head) are exact integers (codes doubled are
// the integers {0,1,2,3,4,6,8,12} with sign), computed on the tensor cores with
// mma.sync.m16n8k32 s8 x s8 -> s32.  A key nibble is turned into its doubled magnitude by one
// PRMT lookup: the code's sign bit is PRMT's sign-replicate flag, so negative codes yield 0;
// the same lookup on the nibbles with flipped signs yields the negative codes' magnitudes, and
// dot = pos . q - neg . q = pos . q + neg . (-q).  B columns 0..3 hold the query heads over
// group 0 and columns 4..7 over group 1, so one accumulator holds both group dots.
// The fp32 score then follows a fixed operation order (see the ABI header), so the selection
// is reproducible bit for bit; order key = (score, -index).
//
// One kernel (indexer_topk_kernel), grid (chunk, sequence), 16 warps per CTA: each CTA streams
// `chunk` entries of keys through shared memory with 1-D bulk copies (3-stage mbarrier ring of
// 512-entry tiles), scores them into 32-bit order keys held in shared memory while building a
// histogram of the keys' top 11 bits, and selects its chunk's top min(k, chunk) -- threshold
// bin from the histogram, one pass to count and collect that bin's candidates, a radix
// select among the candidates only, one pass to emit in index order -- written as a run.  The runs are then merged by a tree inside the same kernel:
// the last CTA of a group of G runs to finish (an atomic arrival counter; nothing ever waits)
// loads the group's runs, selects their top min(k, ...) and publishes one run for the next
// level; the last run is the answer, written in ascending index order and -1 padded.
// Selecting the top k of a union of per-part top-k sets is exact under the total order
// (score desc, index asc), because every global top-k entry is in its part's top k.
#include "csld_internal.cuh"
#include "kernels.cuh"

namespace csld {

constexpr int kIdxThreads = 512;
constexpr int kIdxWarps = kIdxThreads / 32;
constexpr int kIdxTile = 512;          // entries per pipeline stage (32 per warp)
constexpr int kIdxStages = 3;
constexpr int kIdxMaxChunk = 8192;     // keys a CTA holds (chunk, or runs being merged)
constexpr int kIdxMaxGroup = 64;       // runs merged by one CTA
constexpr int kIdxMaxLevels = 4;
constexpr int kBinShift = 21;          // histogram bin = top 11 bits of the order key
constexpr int kBins = 1 << (32 - kBinShift);
constexpr int kRadixBits = 11;
constexpr int kRadixBins = 1 << kRadixBits;

struct IdxSmem {
    union {
        struct {
            uint8_t codes[kIdxStages][kIdxTile * kIkey];
            float scales[kIdxStages][kIdxTile * 2];
        } pipe;                        // key stream ring (scoring)
        struct {
            uint32_t key[kIdxMaxChunk];
            uint16_t pos[kIdxMaxChunk];
        } cand;                        // threshold-bin candidates (selection)
    } u;
    uint32_t keys[kIdxMaxChunk];       // order keys of the chunk, or of the runs being merged
    uint32_t hist[kBins];              // top-11-bit histogram of keys[]
    uint32_t rhist[kRadixBins];        // radix passes over the candidates
    uint32_t wgt[kIdxWarps], wsel[kIdxWarps], weq[kIdxWarps], wbase[kIdxWarps], weqb[kIdxWarps];
    uint32_t red[2 * kIdxWarps];
    int32_t offs[kIdxMaxGroup + 1];
    float qscale[8];                   // [group*4 + head] * 0.25
    uint64_t full[kIdxStages];
    uint32_t sel[4];                   // bin / threshold results
    uint32_t ncand;
    int32_t last;
};

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
__global__ void __launch_bounds__(kIdxThreads) indexer_topk_kernel(
    const uint8_t* __restrict__ ikeys, const float* __restrict__ iscales, int64_t cap,
    const int32_t* __restrict__ seq_len, int ratio, const float* __restrict__ q_idx,
    const float* __restrict__ head_w, int chunk, int kc, int k, IdxTree tree,
    int32_t* __restrict__ topk_out, int32_t* err) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    IdxSmem& sm = *reinterpret_cast<IdxSmem*>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, cq = lane & 3;
    const int b = blockIdx.y, ch = blockIdx.x;

    int64_t n_b = seq_len[b];
    n_b = n_b < 0 ? 0 : n_b / ratio;
    if (n_b > cap) n_b = cap;
    const int64_t c0 = (int64_t)ch * chunk;
    const int cn = static_cast<int>(max64(0, min64(chunk, n_b - c0)));

    for (int i = tid; i < kBins; i += blockDim.x) sm.hist[i] = 0u;
    bool chunk_ok = true;
    if (cn > 0) {
        // --- query: FP4 codes doubled as int8, in the MMA's B layout ----------------------
        // B column n (= g): n < 4 -> head n over group 0; n >= 4 -> head n-4 over group 1.
        // K order inside a group: MMA k = 4c+i <-> dim 8c+i, k = 16+4c+i <-> dim 8c+4+i.
        uint32_t bq0, bq1;
        {
            const int h = g & 3, grp = g >> 2;
            const float* qv = q_idx + ((size_t)b * kIdxHeads + h) * kIdxDim + 32 * grp;
            float amax = 0.f;
            for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(qv[i]));
            const float sg = fp4_group_scale(amax);
            const float inv = 1.0f / sg;   // exact: a power of two
            if (warp == 0 && cq == 0) sm.qscale[grp * 4 + h] = sg;
            uint32_t w0 = 0u, w1 = 0u;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint32_t c_lo = e2m1_code(qv[8 * cq + i] * inv);
                const uint32_t c_hi = e2m1_code(qv[8 * cq + 4 + i] * inv);
                const int v_lo = static_cast<int>(prmt(kTwiceE2M1Lo, kTwiceE2M1Hi, c_lo & 7u) & 0xFFu) *
                                 ((c_lo & 8u) ? -1 : 1);
                const int v_hi = static_cast<int>(prmt(kTwiceE2M1Lo, kTwiceE2M1Hi, c_hi & 7u) & 0xFFu) *
                                 ((c_hi & 8u) ? -1 : 1);
                w0 |= (static_cast<uint32_t>(v_lo) & 0xFFu) << (8 * i);
                w1 |= (static_cast<uint32_t>(v_hi) & 0xFFu) << (8 * i);
            }
            bq0 = w0;
            bq1 = w1;
        }
        // group-0 MMAs see columns 0..3 only, group-1 MMAs columns 4..7 only
        const bool col_grp1 = g >= 4;
        const uint32_t b00 = col_grp1 ? 0u : bq0, b01 = col_grp1 ? 0u : bq1;
        const uint32_t b10 = col_grp1 ? bq0 : 0u, b11 = col_grp1 ? bq1 : 0u;
        auto neg4 = [](uint32_t v) -> uint32_t {   // bytewise negation (|values| <= 12)
            uint32_t r = 0u;
#pragma unroll
            for (int i = 0; i < 4; ++i) r |= ((0u - ((v >> (8 * i)) & 0xFFu)) & 0xFFu) << (8 * i);
            return r;
        };
        const uint32_t n00 = neg4(b00), n01 = neg4(b01), n10 = neg4(b10), n11 = neg4(b11);
        const float w0 = head_w[b * kIdxHeads + 0], w1 = head_w[b * kIdxHeads + 1];
        const float w2 = head_w[b * kIdxHeads + 2], w3 = head_w[b * kIdxHeads + 3];

        if (tid == 0) {
            for (int s = 0; s < kIdxStages; ++s) mbar_init(&sm.full[s], 1);
            fence_barrier_init();
        }
        __syncthreads();
        // query group scales of the two heads this lane finishes
        const int hp = (cq & 1) * 2;
        const float qs0a = sm.qscale[hp], qs0b = sm.qscale[hp + 1];
        const float qs1a = sm.qscale[4 + hp], qs1b = sm.qscale[4 + hp + 1];

        const int n_tiles = (cn + kIdxTile - 1) / kIdxTile;
        const uint8_t* kbase = ikeys + ((size_t)b * cap + (size_t)c0) * kIkey;
        const float* sbase = iscales + ((size_t)b * cap + (size_t)c0) * 2;
        auto issue = [&](int tile) {
            const int s = tile % kIdxStages;
            const int nt = min(kIdxTile, cn - tile * kIdxTile);
            const int nt2 = (nt + 1) & ~1;   // scales copy: a multiple of 16 bytes (cap is even)
            const uint32_t cb = static_cast<uint32_t>(nt) * kIkey;
            const uint32_t sb = static_cast<uint32_t>(nt2) * 8u;
            mbar_arrive_expect_tx(&sm.full[s], cb + sb);
            bulk_g2s(sm.u.pipe.codes[s], kbase + (size_t)tile * kIdxTile * kIkey, cb, &sm.full[s]);
            bulk_g2s(sm.u.pipe.scales[s], sbase + (size_t)tile * kIdxTile * 2, sb, &sm.full[s]);
        };
        if (tid == 0)
            for (int t = 0; t < min(n_tiles, kIdxStages); ++t) issue(t);

        int consumed = 0;
        bool ok = true;
        for (int tile = 0; tile < n_tiles; ++tile) {
            const int s = tile % kIdxStages;
            const bool landed = mbar_wait(&sm.full[s], (tile / kIdxStages) & 1);
            if (__syncthreads_or(!landed)) {
                ok = false;
                break;
            }
            consumed = tile + 1;
            const uint8_t* cs = sm.u.pipe.codes[s];
            const float* ss = sm.u.pipe.scales[s];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int rA = 32 * warp + 16 * half + g, rB = rA + 8;
                const uint32_t kA0 = *reinterpret_cast<const uint32_t*>(cs + rA * kIkey + 4 * cq);
                const uint32_t kB0 = *reinterpret_cast<const uint32_t*>(cs + rB * kIkey + 4 * cq);
                const uint32_t kA1 = *reinterpret_cast<const uint32_t*>(cs + rA * kIkey + 16 + 4 * cq);
                const uint32_t kB1 = *reinterpret_cast<const uint32_t*>(cs + rB * kIkey + 16 + 4 * cq);
                // positive and negative magnitude planes accumulate separately (two MMA chains)
                int accp[4] = {0, 0, 0, 0}, accn[4] = {0, 0, 0, 0};
                auto lut = [](uint32_t sel) { return prmt(kTwiceE2M1Lo, kTwiceE2M1Hi, sel); };
                const uint32_t nA0 = kA0 ^ 0x88888888u, nB0 = kB0 ^ 0x88888888u;
                const uint32_t nA1 = kA1 ^ 0x88888888u, nB1 = kB1 ^ 0x88888888u;
                mma_s8(accp, lut(kA0), lut(kB0), lut(kA0 >> 16), lut(kB0 >> 16), b00, b01);
                mma_s8(accn, lut(nA0), lut(nB0), lut(nA0 >> 16), lut(nB0 >> 16), n00, n01);
                mma_s8(accp, lut(kA1), lut(kB1), lut(kA1 >> 16), lut(kB1 >> 16), b10, b11);
                mma_s8(accn, lut(nA1), lut(nB1), lut(nA1 >> 16), lut(nB1 >> 16), n10, n11);
                int acc[4];
#pragma unroll
                for (int r = 0; r < 4; ++r) acc[r] = accp[r] + accn[r];
                // acc: (row g, cols 2cq, 2cq+1), (row g+8, same).  cq < 2: group-0 dots of
                // heads 2cq, 2cq+1; cq >= 2: group-1 dots of heads 2(cq-2), 2(cq-2)+1.
                const bool lo = cq < 2;
                const int send0 = lo ? acc[2] : acc[0], send1 = lo ? acc[3] : acc[1];
                const int got0 = __shfl_xor_sync(0xffffffffu, send0, 2);
                const int got1 = __shfl_xor_sync(0xffffffffu, send1, 2);
                const int row = lo ? rA : rB;
                const int i0a = lo ? acc[0] : got0, i0b = lo ? acc[1] : got1;
                const int i1a = lo ? got0 : acc[2], i1b = lo ? got1 : acc[3];
                const float ks0 = ss[2 * row], ks1 = ss[2 * row + 1];
                // d = fma(I1, s1, I0*s0) with s_g = (qscale_g * kscale_g) * 0.25
                const float s0a = __fmul_rn(__fmul_rn(qs0a, ks0), 0.25f), s1a = __fmul_rn(__fmul_rn(qs1a, ks1), 0.25f);
                const float s0b = __fmul_rn(__fmul_rn(qs0b, ks0), 0.25f), s1b = __fmul_rn(__fmul_rn(qs1b, ks1), 0.25f);
                const float da = __fmaf_rn(static_cast<float>(i1a), s1a, __fmul_rn(static_cast<float>(i0a), s0a));
                const float db = __fmaf_rn(static_cast<float>(i1b), s1b, __fmul_rn(static_cast<float>(i0b), s0b));
                const float r0 = da > 0.f ? da : 0.f, r1 = db > 0.f ? db : 0.f;
                const float r2 = __shfl_xor_sync(0xffffffffu, r0, 1);
                const float r3 = __shfl_xor_sync(0xffffffffu, r1, 1);
                if ((cq & 1) == 0) {
                    float e = __fmul_rn(w0, r0);
                    e = __fmaf_rn(w1, r1, e);
                    e = __fmaf_rn(w2, r2, e);
                    e = __fmaf_rn(w3, r3, e);
                    const int li = tile * kIdxTile + row;
                    if (li < cn) {
                        const uint32_t key = score_key(e);
                        sm.keys[li] = key;
                        atomicAdd(&sm.hist[key >> kBinShift], 1u);
                    }
                }
            }
            __syncthreads();   // stage s fully consumed
            if (tid == 0 && tile + kIdxStages < n_tiles) issue(tile + kIdxStages);
        }
        chunk_ok = ok;
        if (!ok) {
            // A copy did not land in time: record it, drain what is in flight (bounded), and
            // publish this chunk as empty so the merge tree still completes.
            if (tid == 0) {
                dev_error(err, CSLD_DEVERR_TIMEOUT);
                for (int t = consumed; t < min(n_tiles, consumed + kIdxStages); ++t)
                    (void)mbar_wait(&sm.full[t % kIdxStages], (t / kIdxStages) & 1);
            }
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

cudaError_t launch_indexer(const uint8_t* ikeys, const float* iscales, int64_t cap,
                           const int32_t* seq_len, int ratio, const float* q_idx,
                           const float* head_w, int B, int k, int32_t* topk_out, void* ws,
                           const IndexerPlan& plan, int32_t* err, cudaStream_t stream) {
    size_t bytes = 0;
    IdxTree tree = tree_layout(B, plan.n_chunks, plan.kc, k, plan.group, static_cast<uint8_t*>(ws), &bytes);
    const size_t smem = sizeof(IdxSmem);
    cudaError_t e = set_smem_once(indexer_topk_kernel, smem);
    if (e != cudaSuccess) return e;
    dim3 grid(plan.n_chunks, B);
    indexer_topk_kernel<<<grid, kIdxThreads, smem, stream>>>(ikeys, iscales, cap, seq_len, ratio,
                                                             q_idx, head_w, plan.chunk, plan.kc, k,
                                                             tree, topk_out, err);
    return cudaGetLastError();
}

}  // namespace csld
