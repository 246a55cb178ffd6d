// extern "C" entry points of libcsld: host-side validation, workspace sizing and launches.
// Every check happens before anything is enqueued; a failed check launches nothing.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <set>
#include <utility>

#include "csld_internal.cuh"
#include "kernels.cuh"

namespace csld {
// stage.cu
cudaError_t launch_stage(void* dst, const void* src, size_t bytes, int num_sms, cudaStream_t stream);
// indexer_multi.cu
size_t indexer_multi_ws_bytes(int B, int Q, int64_t cap, int num_sms);
cudaError_t launch_indexer_multi(const uint8_t* ikeys, const float* iscales, int64_t cap, const int32_t* seq_len,
                                 int ratio, const float* q_idx, const float* head_w, int B, int Q, int k,
                                 int32_t* topk_out, void* ws, int num_sms, int32_t* err, cudaStream_t stream,
                                 bool perhead = false);
// cp.cu
cudaError_t launch_indexer_rescore(const uint8_t* ikeys, const float* iscales, int64_t cap, const float* q_idx,
                                   const float* head_w, const int32_t* sel, int B, int k, float* scores,
                                   cudaStream_t stream);
int topk_merge_max_candidates();
cudaError_t launch_topk_merge(const float* cand_score, const int32_t* cand_idx, const int64_t* rank_lo, int R, int B,
                              int k, int64_t lo, int64_t n_local, int32_t* out, cudaStream_t stream);
cudaError_t launch_lse_merge(const float* outs, const float* lses, int R, int BH, float* out, float* lse,
                             cudaStream_t stream);

cudaError_t set_smem_attr_once(const void* kernel, size_t bytes) {
    static std::mutex mu;
    static std::set<std::pair<const void*, int>> done;   // (kernel, device) pairs already set
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    if (done.count({kernel, dev})) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
    if (e == cudaSuccess) done.insert({kernel, dev});
    return e;
}
}  // namespace csld

namespace {

thread_local char g_msg[512] = "";

csld_status fail(csld_status s, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
    va_end(ap);
    return s;
}

csld_status cuda_fail(cudaError_t e, const char* where) {
    return fail(CSLD_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int num_sms() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
    return n;
}

cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

csld_status check_cache(const csld_layer_cache* c) {
    if (!c) return fail(CSLD_ERR_ARG, "cache is NULL");
    if (c->ratio < 1 || c->ratio > CSLD_MAX_RATIO)
        return fail(CSLD_ERR_ARG, "ratio %d outside 1..%d", c->ratio, CSLD_MAX_RATIO);
    if (c->window < 0 || c->window > CSLD_MAX_WINDOW)
        return fail(CSLD_ERR_ARG, "window %d outside 0..%d", c->window, CSLD_MAX_WINDOW);
    if (c->batch < 1 || c->batch > 65535) return fail(CSLD_ERR_ARG, "batch %d outside 1..65535", c->batch);
    if (c->capacity < 1 || c->capacity > (int64_t)INT32_MAX)
        return fail(CSLD_ERR_ARG, "capacity %lld outside 1..2^31-1", (long long)c->capacity);
    if (!c->comp_kv || !c->tail_kv || !c->tail_gate || !c->seq_len || !c->pos_bias)
        return fail(CSLD_ERR_ARG, "a required cache pointer is NULL");
    if (c->window > 0 && !c->win_kv) return fail(CSLD_ERR_ARG, "win_kv is NULL with window > 0");
    if (c->has_indexer && (!c->ikeys || !c->iscales || !c->w_idx))
        return fail(CSLD_ERR_ARG, "indexer arrays are NULL with has_indexer set");
    if (c->has_indexer && (c->capacity & 1))
        return fail(CSLD_ERR_ALIGN, "capacity must be even when the cache keeps indexer keys");
    if (!aligned16(c->comp_kv) || (c->win_kv && !aligned16(c->win_kv)) || !aligned16(c->tail_kv) ||
        (c->ikeys && !aligned16(c->ikeys)) || (c->iscales && !aligned16(c->iscales)))
        return fail(CSLD_ERR_ALIGN, "cache arrays must be 16-byte aligned");
    return CSLD_OK;
}

}  // namespace

extern "C" {

int csld_abi_version(void) { return CSLD_ABI_VERSION; }

const char* csld_last_error(void) { return g_msg; }

const char* csld_status_string(csld_status s) {
    switch (s) {
        case CSLD_OK: return "ok";
        case CSLD_ERR_ARG: return "invalid argument";
        case CSLD_ERR_SHAPE: return "inconsistent shape";
        case CSLD_ERR_ALIGN: return "misaligned pointer or stride";
        case CSLD_ERR_CAPACITY: return "size exceeds a maximum or the cache capacity";
        case CSLD_ERR_CUDA: return "CUDA error";
        case CSLD_ERR_UNSUPPORTED: return "unsupported shape";
        case CSLD_ERR_WORKSPACE: return "workspace missing or too small";
    }
    return "unknown status";
}

namespace {
csld_status compress_impl(const char* name, const uint16_t* raw, const float* gate, const float* pos_bias, int ratio,
                          const float* w_idx, int64_t T, int64_t pos0, double rope_base, float kv_scale,
                          uint8_t* kv_out, uint8_t* ikey_out, float* iscale_out, void* stream, bool perhead = false) {
    if (ratio < 1 || ratio > CSLD_MAX_RATIO) return fail(CSLD_ERR_ARG, "ratio %d outside 1..%d", ratio, CSLD_MAX_RATIO);
    if (T < 0 || T > (int64_t)INT32_MAX) return fail(CSLD_ERR_ARG, "T %lld outside 0..2^31-1", (long long)T);
    if (T / ratio == 0) return CSLD_OK;
    if (!raw || !gate || !pos_bias || !kv_out) return fail(CSLD_ERR_ARG, "a required pointer is NULL");
    if (w_idx && (!ikey_out || !iscale_out)) return fail(CSLD_ERR_ARG, "ikey_out / iscale_out NULL with w_idx");
    if (!aligned16(raw) || !aligned16(kv_out) || (ikey_out && !aligned16(ikey_out)))
        return fail(CSLD_ERR_ALIGN, "raw, kv_out and ikey_out must be 16-byte aligned");
    cudaError_t e = csld::launch_compress(raw, gate, pos_bias, ratio, w_idx, T, 1, T / ratio, kv_out,
                                          ikey_out, iscale_out, num_sms(), as_stream(stream), pos0, rope_base,
                                          kv_scale, perhead);
    if (e != cudaSuccess) return cuda_fail(e, name);
    return CSLD_OK;
}
}  // namespace

csld_status csld_compress(const uint16_t* raw, const float* gate, const float* pos_bias, int ratio,
                          const float* w_idx, int64_t T, uint8_t* kv_out, uint8_t* ikey_out,
                          float* iscale_out, void* stream) {
    return compress_impl("csld_compress", raw, gate, pos_bias, ratio, w_idx, T, 0, 0.0, 1.f, kv_out, ikey_out,
                         iscale_out, stream);
}

csld_status csld_compress_rope(const uint16_t* raw, const float* gate, const float* pos_bias, int ratio,
                               const float* w_idx, int64_t T, int64_t pos0, double rope_base, uint8_t* kv_out,
                               uint8_t* ikey_out, float* iscale_out, void* stream) {
    if (!(rope_base > 1.0) || rope_base == INFINITY) return fail(CSLD_ERR_ARG, "rope_base must be finite and > 1");
    if (pos0 < 0 || pos0 > ((int64_t)1 << 40)) return fail(CSLD_ERR_ARG, "pos0 %lld outside 0..2^40", (long long)pos0);
    return compress_impl("csld_compress_rope", raw, gate, pos_bias, ratio, w_idx, T, pos0, rope_base, 1.f, kv_out,
                         ikey_out, iscale_out, stream);
}

namespace {
bool kv_scale_ok(float kv_scale) { return kv_scale >= 0x1p-60f && kv_scale <= 0x1p60f; }
}  // namespace

csld_status csld_compress_perhead(const uint16_t* raw, const float* gate, const float* pos_bias, int ratio,
                                  const float* w_idx, int64_t T, uint8_t* kv_out, uint8_t* ikey_out, float* iscale_out,
                                  void* stream) {
    if (!w_idx) return fail(CSLD_ERR_ARG, "w_idx is NULL (per-head keys need the projection)");
    return compress_impl("csld_compress_perhead", raw, gate, pos_bias, ratio, w_idx, T, 0, 0.0, 1.f, kv_out, ikey_out,
                         iscale_out, stream, true);
}

csld_status csld_compress_scaled(const uint16_t* raw, const float* gate, const float* pos_bias, int ratio,
                                 const float* w_idx, int64_t T, float kv_scale, uint8_t* kv_out, uint8_t* ikey_out,
                                 float* iscale_out, void* stream) {
    if (!kv_scale_ok(kv_scale)) return fail(CSLD_ERR_ARG, "kv_scale %g outside 2^-60..2^60", (double)kv_scale);
    return compress_impl("csld_compress_scaled", raw, gate, pos_bias, ratio, w_idx, T, 0, 0.0, kv_scale, kv_out,
                         ikey_out, iscale_out, stream);
}

csld_status csa_compress(const uint16_t* raw, const float* gate, const float* pos_bias,
                         const float* w_idx, int64_t T, uint8_t* kv_out, uint8_t* ikey_out,
                         float* iscale_out, void* stream) {
    if (!w_idx) return fail(CSLD_ERR_ARG, "csa_compress needs w_idx");
    return csld_compress(raw, gate, pos_bias, 4, w_idx, T, kv_out, ikey_out, iscale_out, stream);
}

csld_status hca_compress(const uint16_t* raw, const float* gate, const float* pos_bias, int64_t T,
                         uint8_t* kv_out, void* stream) {
    return csld_compress(raw, gate, pos_bias, 128, nullptr, T, kv_out, nullptr, nullptr, stream);
}

namespace {
csld_status append_impl(const char* name, const csld_layer_cache* cache, const uint16_t* kv_new,
                        const float* gate_new, int32_t* err, double rope_base, float kv_scale, void* stream,
                        bool perhead = false) {
    csld_status s = check_cache(cache);
    if (s != CSLD_OK) return s;
    if (!kv_new || !gate_new) return fail(CSLD_ERR_ARG, "kv_new / gate_new is NULL");
    if (!aligned16(kv_new)) return fail(CSLD_ERR_ALIGN, "kv_new must be 16-byte aligned");
    cudaError_t e = csld::launch_append(*cache, kv_new, gate_new, err, as_stream(stream), rope_base, kv_scale, perhead);
    if (e != cudaSuccess) return cuda_fail(e, name);
    return CSLD_OK;
}
}  // namespace

csld_status kv_cache_append(const csld_layer_cache* cache, const uint16_t* kv_new,
                            const float* gate_new, int32_t* err, void* stream) {
    return append_impl("kv_cache_append", cache, kv_new, gate_new, err, 0.0, 1.f, stream);
}

csld_status kv_cache_append_rope(const csld_layer_cache* cache, const uint16_t* kv_new,
                                 const float* gate_new, double rope_base, int32_t* err, void* stream) {
    if (!(rope_base > 1.0) || rope_base == INFINITY) return fail(CSLD_ERR_ARG, "rope_base must be finite and > 1");
    return append_impl("kv_cache_append_rope", cache, kv_new, gate_new, err, rope_base, 1.f, stream);
}

csld_status kv_cache_append_perhead(const csld_layer_cache* cache, const uint16_t* kv_new,
                                    const float* gate_new, int32_t* err, void* stream) {
    if (!cache || !cache->has_indexer) return fail(CSLD_ERR_ARG, "per-head keys need a cache with an indexer");
    return append_impl("kv_cache_append_perhead", cache, kv_new, gate_new, err, 0.0, 1.f, stream, true);
}

csld_status kv_cache_append_scaled(const csld_layer_cache* cache, const uint16_t* kv_new,
                                   const float* gate_new, float kv_scale, int32_t* err, void* stream) {
    if (!kv_scale_ok(kv_scale)) return fail(CSLD_ERR_ARG, "kv_scale %g outside 2^-60..2^60", (double)kv_scale);
    return append_impl("kv_cache_append_scaled", cache, kv_new, gate_new, err, 0.0, kv_scale, stream);
}

namespace {
csld_status prefill_impl(const csld_layer_cache* cache, const uint16_t* raw, const float* gate, int64_t T,
                         double rope_base, float kv_scale, void* stream, bool perhead = false) {
    csld_status s = check_cache(cache);
    if (s != CSLD_OK) return s;
    if (T < 0 || T > (int64_t)INT32_MAX) return fail(CSLD_ERR_ARG, "T %lld outside 0..2^31-1", (long long)T);
    if (T > 0 && (!raw || !gate)) return fail(CSLD_ERR_ARG, "raw / gate is NULL");
    if (T > 0 && !aligned16(raw)) return fail(CSLD_ERR_ALIGN, "raw must be 16-byte aligned");
    if (T / cache->ratio > cache->capacity)
        return fail(CSLD_ERR_CAPACITY, "T/ratio = %lld entries exceed capacity %lld",
                    (long long)(T / cache->ratio), (long long)cache->capacity);
    const cudaStream_t st = as_stream(stream);
    cudaError_t e = csld::launch_compress(raw, gate, cache->pos_bias, cache->ratio,
                                          cache->has_indexer ? cache->w_idx : nullptr, T, cache->batch,
                                          cache->capacity, cache->comp_kv, cache->ikeys,
                                          cache->iscales, num_sms(), st, 0, rope_base, kv_scale, perhead);
    if (e != cudaSuccess) return cuda_fail(e, "kv_cache_prefill (compress)");
    e = csld::launch_prefill_state(raw, gate, T, cache->ratio, cache->window, cache->batch,
                                   cache->win_kv, cache->tail_kv, cache->tail_gate, cache->seq_len, st, rope_base,
                                   kv_scale);
    if (e != cudaSuccess) return cuda_fail(e, "kv_cache_prefill (state)");
    return CSLD_OK;
}
}  // namespace

csld_status kv_cache_prefill(const csld_layer_cache* cache, const uint16_t* raw, const float* gate,
                             int64_t T, void* stream) {
    return prefill_impl(cache, raw, gate, T, 0.0, 1.f, stream);
}

csld_status kv_cache_prefill_rope(const csld_layer_cache* cache, const uint16_t* raw, const float* gate,
                                  int64_t T, double rope_base, void* stream) {
    if (!(rope_base > 1.0) || rope_base == INFINITY) return fail(CSLD_ERR_ARG, "rope_base must be finite and > 1");
    return prefill_impl(cache, raw, gate, T, rope_base, 1.f, stream);
}

csld_status kv_cache_prefill_perhead(const csld_layer_cache* cache, const uint16_t* raw, const float* gate,
                                     int64_t T, void* stream) {
    if (!cache || !cache->has_indexer) return fail(CSLD_ERR_ARG, "per-head keys need a cache with an indexer");
    return prefill_impl(cache, raw, gate, T, 0.0, 1.f, stream, true);
}

csld_status kv_cache_prefill_scaled(const csld_layer_cache* cache, const uint16_t* raw, const float* gate,
                                    int64_t T, float kv_scale, void* stream) {
    if (!kv_scale_ok(kv_scale)) return fail(CSLD_ERR_ARG, "kv_scale %g outside 2^-60..2^60", (double)kv_scale);
    return prefill_impl(cache, raw, gate, T, 0.0, kv_scale, stream);
}

size_t csld_indexer_workspace_size(int B, int64_t cap, int k) {
    if (B < 1 || cap < 1 || k < 1) return 0;
    return csld::indexer_plan(B, cap, k, num_sms()).ws_bytes;
}

csld_status indexer_topk(const uint8_t* ikeys, const float* iscales, int64_t cap,
                         const int32_t* seq_len, int ratio, const float* q_idx, const float* head_w,
                         int B, int k, int32_t* topk_out, void* ws, size_t ws_bytes, int32_t* err,
                         void* stream) {
    if (B < 1 || B > 65535) return fail(CSLD_ERR_ARG, "B %d outside 1..65535", B);
    if (k < 1 || k > CSLD_MAX_TOPK) return fail(CSLD_ERR_ARG, "k %d outside 1..%d", k, CSLD_MAX_TOPK);
    if (cap < 1 || cap > ((int64_t)1 << 30)) return fail(CSLD_ERR_ARG, "cap %lld outside 1..2^30", (long long)cap);
    if (cap & 1) return fail(CSLD_ERR_ALIGN, "cap must be even");
    if (ratio < 1 || ratio > CSLD_MAX_RATIO) return fail(CSLD_ERR_ARG, "ratio %d outside 1..%d", ratio, CSLD_MAX_RATIO);
    if (!ikeys || !iscales || !seq_len || !q_idx || !head_w || !topk_out)
        return fail(CSLD_ERR_ARG, "a required pointer is NULL");
    if (!aligned16(ikeys) || !aligned16(iscales)) return fail(CSLD_ERR_ALIGN, "ikeys / iscales must be 16-byte aligned");
    const csld::IndexerPlan plan = csld::indexer_plan(B, cap, k, num_sms());
    if (!plan.levels_ok) return fail(CSLD_ERR_CAPACITY, "cap %lld too large for the merge tree", (long long)cap);
    if (!ws || ws_bytes < plan.ws_bytes)
        return fail(CSLD_ERR_WORKSPACE, "workspace %zu bytes < required %zu", ws_bytes, plan.ws_bytes);
    if (reinterpret_cast<uintptr_t>(ws) & 255u) return fail(CSLD_ERR_ALIGN, "workspace must be 256-byte aligned");
    cudaError_t e = csld::launch_indexer(ikeys, iscales, cap, seq_len, ratio, q_idx, head_w, B, k,
                                         topk_out, ws, plan, err, as_stream(stream));
    if (e != cudaSuccess) return cuda_fail(e, "indexer_topk");
    return CSLD_OK;
}

size_t csld_attention_workspace_size(int B, int heads, int64_t cap, int k, int W) {
    if (B < 1 || heads != CSLD_HEADS || cap < 1 || W < 0) return 0;
    const csld::AttentionPlan pd = csld::attention_plan(B, cap, k, false, W, num_sms());
    const csld::AttentionPlan ps = csld::attention_plan(B, cap, k > 0 ? k : 1, true, W, num_sms());
    return pd.ws_bytes > ps.ws_bytes ? pd.ws_bytes : ps.ws_bytes;
}

namespace {
csld_status attention_impl(const char* name, const uint16_t* q, int heads, const uint8_t* comp_kv, int64_t cap,
                           int ratio, const int32_t* topk, int k, const uint8_t* win_kv, int W,
                           const int32_t* seq_len, int B, float scale, float kv_scale, float* out, float* lse_out,
                           void* ws, size_t ws_bytes, int32_t* err, void* stream) {
    if (heads != CSLD_HEADS) return fail(CSLD_ERR_UNSUPPORTED, "heads = %d; the library implements %d", heads, CSLD_HEADS);
    if (B < 1 || B > 65535) return fail(CSLD_ERR_ARG, "B %d outside 1..65535", B);
    if (cap < 1 || cap > (int64_t)INT32_MAX) return fail(CSLD_ERR_ARG, "cap %lld outside 1..2^31-1", (long long)cap);
    if (ratio < 1 || ratio > CSLD_MAX_RATIO) return fail(CSLD_ERR_ARG, "ratio %d outside 1..%d", ratio, CSLD_MAX_RATIO);
    if (W < 0 || W > CSLD_MAX_WINDOW) return fail(CSLD_ERR_ARG, "W %d outside 0..%d", W, CSLD_MAX_WINDOW);
    if (topk && (k < 1 || k > CSLD_MAX_TOPK)) return fail(CSLD_ERR_ARG, "k %d outside 1..%d", k, CSLD_MAX_TOPK);
    if (!(scale == scale) || scale == INFINITY || scale == -INFINITY) return fail(CSLD_ERR_ARG, "scale is not finite");
    if (!q || !comp_kv || !seq_len || !out) return fail(CSLD_ERR_ARG, "a required pointer is NULL");
    if (W > 0 && !win_kv) return fail(CSLD_ERR_ARG, "win_kv is NULL with W > 0");
    if (!aligned16(q) || !aligned16(comp_kv) || (win_kv && !aligned16(win_kv)) || !aligned16(out))
        return fail(CSLD_ERR_ALIGN, "q, comp_kv, win_kv and out must be 16-byte aligned");
    const csld::AttentionPlan plan = csld::attention_plan(B, cap, k, topk != nullptr, W, num_sms());
    if (!ws || ws_bytes < plan.ws_bytes)
        return fail(CSLD_ERR_WORKSPACE, "workspace %zu bytes < required %zu", ws_bytes, plan.ws_bytes);
    if (!aligned16(ws)) return fail(CSLD_ERR_ALIGN, "workspace must be 16-byte aligned");
    cudaError_t e = csld::launch_attention(q, comp_kv, cap, ratio, topk, topk ? k : 0, win_kv, W, W, 1, seq_len, B,
                                           scale, out, lse_out, ws, plan, err, as_stream(stream), kv_scale);
    if (e != cudaSuccess) return cuda_fail(e, name);
    return CSLD_OK;
}
}  // namespace

csld_status hybrid_decode_attention(const uint16_t* q, int heads, const uint8_t* comp_kv, int64_t cap,
                                    int ratio, const int32_t* topk, int k, const uint8_t* win_kv, int W,
                                    const int32_t* seq_len, int B, float scale, float* out, float* lse_out,
                                    void* ws, size_t ws_bytes, int32_t* err, void* stream) {
    return attention_impl("hybrid_decode_attention", q, heads, comp_kv, cap, ratio, topk, k, win_kv, W, seq_len, B,
                          scale, 1.f, out, lse_out, ws, ws_bytes, err, stream);
}

csld_status hybrid_decode_attention_scaled(const uint16_t* q, int heads, const uint8_t* comp_kv, int64_t cap,
                                           int ratio, const int32_t* topk, int k, const uint8_t* win_kv, int W,
                                           const int32_t* seq_len, int B, float scale, float kv_scale, float* out,
                                           float* lse_out, void* ws, size_t ws_bytes, int32_t* err, void* stream) {
    if (!kv_scale_ok(kv_scale)) return fail(CSLD_ERR_ARG, "kv_scale %g outside 2^-60..2^60", (double)kv_scale);
    return attention_impl("hybrid_decode_attention_scaled", q, heads, comp_kv, cap, ratio, topk, k, win_kv, W,
                          seq_len, B, scale, kv_scale, out, lse_out, ws, ws_bytes, err, stream);
}

csld_status csld_stage(void* dst, const void* src, size_t bytes, void* stream) {
    if (bytes == 0) return CSLD_OK;
    if (!dst || !src) return fail(CSLD_ERR_ARG, "a required pointer is NULL");
    if (!aligned16(dst) || !aligned16(src) || (bytes & 15u))
        return fail(CSLD_ERR_ALIGN, "dst and src must be 16-byte aligned and bytes a multiple of 16");
    cudaError_t e = csld::launch_stage(dst, src, bytes, num_sms(), as_stream(stream));
    if (e != cudaSuccess) return cuda_fail(e, "csld_stage");
    return CSLD_OK;
}

csld_status hybrid_decode_attention_static(const uint16_t* q, int heads, const uint8_t* comp_kv,
                                           int64_t cap, int ratio, const int32_t* topk, int k,
                                           const uint8_t* win_kv, int W, const int32_t* seq_len, int B,
                                           float scale, float* out, float* lse_out, int32_t* err,
                                           void* stream) {
    if (heads != CSLD_HEADS) return fail(CSLD_ERR_UNSUPPORTED, "heads = %d; the library implements %d", heads, CSLD_HEADS);
    if (B < 1 || B > 65535) return fail(CSLD_ERR_ARG, "B %d outside 1..65535", B);
    if (cap < 1 || cap > (int64_t)INT32_MAX) return fail(CSLD_ERR_ARG, "cap %lld outside 1..2^31-1", (long long)cap);
    if (ratio < 1 || ratio > CSLD_MAX_RATIO) return fail(CSLD_ERR_ARG, "ratio %d outside 1..%d", ratio, CSLD_MAX_RATIO);
    if (W < 0 || W > CSLD_MAX_WINDOW) return fail(CSLD_ERR_ARG, "W %d outside 0..%d", W, CSLD_MAX_WINDOW);
    if (topk && (k < 1 || k > CSLD_MAX_TOPK)) return fail(CSLD_ERR_ARG, "k %d outside 1..%d", k, CSLD_MAX_TOPK);
    if (!(scale == scale) || scale == INFINITY || scale == -INFINITY) return fail(CSLD_ERR_ARG, "scale is not finite");
    if (!q || !comp_kv || !seq_len || !out) return fail(CSLD_ERR_ARG, "a required pointer is NULL");
    if (W > 0 && !win_kv) return fail(CSLD_ERR_ARG, "win_kv is NULL with W > 0");
    if (!aligned16(q) || !aligned16(comp_kv) || (win_kv && !aligned16(win_kv)) || !aligned16(out))
        return fail(CSLD_ERR_ALIGN, "q, comp_kv, win_kv and out must be 16-byte aligned");
    const csld::AttentionPlan plan = csld::attention_plan(B, cap, k, topk != nullptr, W, num_sms());
    if (plan.ws_bytes > (size_t)CSLD_STATIC_SCRATCH_BYTES)
        return fail(CSLD_ERR_CAPACITY,
                    "this call needs %zu bytes of scratch; the library-owned scratch holds %zu bytes "
                    "(use hybrid_decode_attention with a workspace, or a smaller batch)",
                    plan.ws_bytes, (size_t)CSLD_STATIC_SCRATCH_BYTES);
    void* ws = nullptr;
    cudaError_t e = csld::attention_static_scratch(&ws);
    if (e != cudaSuccess) return cuda_fail(e, "hybrid_decode_attention_static (scratch address)");
    e = csld::launch_attention(q, comp_kv, cap, ratio, topk, topk ? k : 0, win_kv, W, W, 1, seq_len, B, scale, out,
                               lse_out, ws, plan, err, as_stream(stream));
    if (e != cudaSuccess) return cuda_fail(e, "hybrid_decode_attention_static");
    return CSLD_OK;
}

csld_status indexer_rescore(const uint8_t* ikeys, const float* iscales, int64_t cap, const float* q_idx,
                            const float* head_w, const int32_t* sel, int B, int k, float* scores_out,
                            void* stream) {
    if (B < 1 || B > 65535) return fail(CSLD_ERR_ARG, "B %d outside 1..65535", B);
    if (k < 1 || k > CSLD_MAX_TOPK) return fail(CSLD_ERR_ARG, "k %d outside 1..%d", k, CSLD_MAX_TOPK);
    if (cap < 1 || cap > ((int64_t)1 << 30)) return fail(CSLD_ERR_ARG, "cap %lld outside 1..2^30", (long long)cap);
    if (cap & 1) return fail(CSLD_ERR_ALIGN, "cap must be even");
    if (!ikeys || !iscales || !q_idx || !head_w || !sel || !scores_out)
        return fail(CSLD_ERR_ARG, "a required pointer is NULL");
    if (!aligned16(iscales)) return fail(CSLD_ERR_ALIGN, "iscales must be 16-byte aligned");
    cudaError_t e = csld::launch_indexer_rescore(ikeys, iscales, cap, q_idx, head_w, sel, B, k, scores_out,
                                                 as_stream(stream));
    if (e != cudaSuccess) return cuda_fail(e, "indexer_rescore");
    return CSLD_OK;
}

csld_status csld_topk_merge(const float* cand_scores, const int32_t* cand_idx, const int64_t* rank_lo, int R, int B,
                            int k, int64_t lo, int64_t n_local, int32_t* topk_out, void* stream) {
    if (B < 1 || B > 65535) return fail(CSLD_ERR_ARG, "B %d outside 1..65535", B);
    if (k < 1 || k > CSLD_MAX_TOPK) return fail(CSLD_ERR_ARG, "k %d outside 1..%d", k, CSLD_MAX_TOPK);
    if (R < 1 || (int64_t)R * k > csld::topk_merge_max_candidates())
        return fail(CSLD_ERR_CAPACITY, "R * k = %lld candidates; at most %d", (long long)R * k,
                    csld::topk_merge_max_candidates());
    if (lo < 0 || n_local < 0 || lo + n_local > ((int64_t)1 << 30))
        return fail(CSLD_ERR_ARG, "local range [%lld, %lld) outside 0..2^30", (long long)lo, (long long)(lo + n_local));
    if (!cand_scores || !cand_idx || !rank_lo || !topk_out) return fail(CSLD_ERR_ARG, "a required pointer is NULL");
    cudaError_t e = csld::launch_topk_merge(cand_scores, cand_idx, rank_lo, R, B, k, lo, n_local, topk_out,
                                            as_stream(stream));
    if (e != cudaSuccess) return cuda_fail(e, "csld_topk_merge");
    return CSLD_OK;
}

csld_status csld_lse_merge(const float* outs, const float* lses, int R, int B, int heads, float* out,
                           float* lse_out, void* stream) {
    if (heads != CSLD_HEADS) return fail(CSLD_ERR_UNSUPPORTED, "heads = %d; the library implements %d", heads, CSLD_HEADS);
    if (B < 1 || B > 65535 || R < 1) return fail(CSLD_ERR_ARG, "B %d or R %d out of range", B, R);
    if (!outs || !lses || !out) return fail(CSLD_ERR_ARG, "a required pointer is NULL");
    if (!aligned16(outs) || !aligned16(out)) return fail(CSLD_ERR_ALIGN, "outs and out must be 16-byte aligned");
    cudaError_t e = csld::launch_lse_merge(outs, lses, R, B * heads, out, lse_out, as_stream(stream));
    if (e != cudaSuccess) return cuda_fail(e, "csld_lse_merge");
    return CSLD_OK;
}

size_t csld_indexer_multi_workspace_size(int B, int Q, int64_t cap) {
    if (B < 1 || Q < 1 || Q > CSLD_MULTI_MAX_Q || cap < 1) return 0;
    return csld::indexer_multi_ws_bytes(B, Q, cap, num_sms());
}

namespace {
csld_status indexer_multi_impl(const char* name, const uint8_t* ikeys, const float* iscales, int64_t cap,
                               const int32_t* seq_len, int ratio, const float* q_idx, const float* head_w, int B, int Q,
                               int k, int32_t* topk_out, void* ws, size_t ws_bytes, int32_t* err, void* stream,
                               bool perhead) {
    if (B < 1 || B > 65535) return fail(CSLD_ERR_ARG, "B %d outside 1..65535", B);
    if (Q < 1 || Q > CSLD_MULTI_MAX_Q) return fail(CSLD_ERR_ARG, "Q %d outside 1..%d", Q, CSLD_MULTI_MAX_Q);
    if (k < 1 || k > CSLD_MAX_TOPK) return fail(CSLD_ERR_ARG, "k %d outside 1..%d", k, CSLD_MAX_TOPK);
    if (cap < 2 || cap > ((int64_t)1 << 30)) return fail(CSLD_ERR_ARG, "cap %lld outside 2..2^30", (long long)cap);
    if (cap & 1) return fail(CSLD_ERR_ALIGN, "cap must be even");
    if (ratio < 1 || ratio > CSLD_MAX_RATIO) return fail(CSLD_ERR_ARG, "ratio %d outside 1..%d", ratio, CSLD_MAX_RATIO);
    if (!ikeys || !iscales || !seq_len || !q_idx || !head_w || !topk_out)
        return fail(CSLD_ERR_ARG, "a required pointer is NULL");
    if (!aligned16(ikeys) || !aligned16(iscales)) return fail(CSLD_ERR_ALIGN, "ikeys / iscales must be 16-byte aligned");
    const size_t need = csld::indexer_multi_ws_bytes(B, Q, cap, num_sms());
    if (!ws || ws_bytes < need) return fail(CSLD_ERR_WORKSPACE, "workspace %zu bytes < required %zu", ws_bytes, need);
    if (reinterpret_cast<uintptr_t>(ws) & 255u) return fail(CSLD_ERR_ALIGN, "workspace must be 256-byte aligned");
    cudaError_t e = csld::launch_indexer_multi(ikeys, iscales, cap, seq_len, ratio, q_idx, head_w, B, Q, k, topk_out,
                                               ws, num_sms(), err, as_stream(stream), perhead);
    if (e != cudaSuccess) return cuda_fail(e, name);
    return CSLD_OK;
}
}  // namespace

csld_status indexer_topk_multi(const uint8_t* ikeys, const float* iscales, int64_t cap, const int32_t* seq_len,
                               int ratio, const float* q_idx, const float* head_w, int B, int Q, int k,
                               int32_t* topk_out, void* ws, size_t ws_bytes, int32_t* err, void* stream) {
    return indexer_multi_impl("indexer_topk_multi", ikeys, iscales, cap, seq_len, ratio, q_idx, head_w, B, Q, k,
                              topk_out, ws, ws_bytes, err, stream, false);
}

csld_status indexer_topk_perhead(const uint8_t* ikeys, const float* iscales, int64_t cap, const int32_t* seq_len,
                                 int ratio, const float* q_idx, const float* head_w, int B, int Q, int k,
                                 int32_t* topk_out, void* ws, size_t ws_bytes, int32_t* err, void* stream) {
    return indexer_multi_impl("indexer_topk_perhead", ikeys, iscales, cap, seq_len, ratio, q_idx, head_w, B, Q, k,
                              topk_out, ws, ws_bytes, err, stream, true);
}

csld_status hybrid_decode_attention_multi(const uint16_t* q, int heads, const uint8_t* comp_kv, int64_t cap,
                                          int ratio, const int32_t* topk, int k, const uint8_t* win_kv, int W_ring,
                                          int W, const int32_t* seq_len, int B, int Q, float scale, float* out,
                                          float* lse_out, void* ws, size_t ws_bytes, int32_t* err, void* stream) {
    if (heads != CSLD_HEADS) return fail(CSLD_ERR_UNSUPPORTED, "heads = %d; the library implements %d", heads, CSLD_HEADS);
    if (B < 1 || Q < 1 || Q > CSLD_MULTI_MAX_Q || (int64_t)B * Q > 65535)
        return fail(CSLD_ERR_ARG, "B %d, Q %d: need 1 <= Q <= %d and B * Q <= 65535", B, Q, CSLD_MULTI_MAX_Q);
    if (cap < 1 || cap > (int64_t)INT32_MAX) return fail(CSLD_ERR_ARG, "cap %lld outside 1..2^31-1", (long long)cap);
    if (ratio < 1 || ratio > CSLD_MAX_RATIO) return fail(CSLD_ERR_ARG, "ratio %d outside 1..%d", ratio, CSLD_MAX_RATIO);
    if (W < 0 || W > CSLD_MAX_WINDOW) return fail(CSLD_ERR_ARG, "W %d outside 0..%d", W, CSLD_MAX_WINDOW);
    if (W > 0 && (W_ring < W + Q - 1 || W_ring > CSLD_MAX_WINDOW + CSLD_MULTI_MAX_Q))
        return fail(CSLD_ERR_ARG, "W_ring %d: need W + Q - 1 = %d <= W_ring <= %d", W_ring, W + Q - 1,
                    CSLD_MAX_WINDOW + CSLD_MULTI_MAX_Q);
    if (topk && (k < 1 || k > CSLD_MAX_TOPK)) return fail(CSLD_ERR_ARG, "k %d outside 1..%d", k, CSLD_MAX_TOPK);
    if (!(scale == scale) || scale == INFINITY || scale == -INFINITY) return fail(CSLD_ERR_ARG, "scale is not finite");
    if (!q || !comp_kv || !seq_len || !out) return fail(CSLD_ERR_ARG, "a required pointer is NULL");
    if (W > 0 && !win_kv) return fail(CSLD_ERR_ARG, "win_kv is NULL with W > 0");
    if (!aligned16(q) || !aligned16(comp_kv) || (win_kv && !aligned16(win_kv)) || !aligned16(out))
        return fail(CSLD_ERR_ALIGN, "q, comp_kv, win_kv and out must be 16-byte aligned");
    const csld::AttentionPlan plan = csld::attention_plan(B * Q, cap, k, topk != nullptr, W, num_sms());
    if (!ws || ws_bytes < plan.ws_bytes)
        return fail(CSLD_ERR_WORKSPACE, "workspace %zu bytes < required %zu", ws_bytes, plan.ws_bytes);
    if (!aligned16(ws)) return fail(CSLD_ERR_ALIGN, "workspace must be 16-byte aligned");
    cudaError_t e = csld::launch_attention(q, comp_kv, cap, ratio, topk, topk ? k : 0, win_kv, W, W > 0 ? W_ring : 0,
                                           Q, seq_len, B, scale, out, lse_out, ws, plan, err, as_stream(stream));
    if (e != cudaSuccess) return cuda_fail(e, "hybrid_decode_attention_multi");
    return CSLD_OK;
}

void csld_test_set_barrier_extra(int extra) { csld::g_test_barrier_extra.store(extra < 0 ? 0 : extra); }

csld_status csld_compress_channel(const uint16_t* raw, const float* gate, const float* pos_bias, int ratio,
                                  const float* w_idx, int64_t T, uint8_t* kv_out, uint8_t* ikey_out,
                                  float* iscale_out, void* stream) {
    if (ratio < 1 || ratio > CSLD_MAX_RATIO) return fail(CSLD_ERR_ARG, "ratio %d outside 1..%d", ratio, CSLD_MAX_RATIO);
    if (T < 0 || T > (int64_t)INT32_MAX) return fail(CSLD_ERR_ARG, "T %lld outside 0..2^31-1", (long long)T);
    if (T / ratio == 0) return CSLD_OK;
    if (!raw || !gate || !pos_bias || !kv_out) return fail(CSLD_ERR_ARG, "a required pointer is NULL");
    if (w_idx && (!ikey_out || !iscale_out)) return fail(CSLD_ERR_ARG, "ikey_out / iscale_out NULL with w_idx");
    if (!aligned16(raw) || !aligned16(gate) || !aligned16(pos_bias) || !aligned16(kv_out) ||
        (ikey_out && !aligned16(ikey_out)))
        return fail(CSLD_ERR_ALIGN, "raw, gate, pos_bias, kv_out and ikey_out must be 16-byte aligned");
    cudaError_t e = csld::launch_compress_channel(raw, gate, pos_bias, ratio, w_idx, T, kv_out, ikey_out, iscale_out,
                                                  num_sms(), as_stream(stream));
    if (e != cudaSuccess) return cuda_fail(e, "csld_compress_channel");
    return CSLD_OK;
}

}  // extern "C"
