// Launchers of the libcsld kernels (host side, internal).
#pragma once
#include <cuda_runtime.h>

#include <atomic>
#include <stdint.h>

#include "csld.h"

namespace csld {

// Layout variants (at most one at a time): rope_base > 0, RoPE at compressed positions with raw
// token 0 at position pos0 (entry s rotated at pos0 + (s+1) m - 1); kv_scale != 1, scaled FP8
// entries (E4M3(x / kv_scale)); perhead, per-head indexer keys (w_idx [512][4][64], keys
// [..][128 B] swizzled, scales [..][4][2]).  rope_base = 0, kv_scale = 1, !perhead: the base layout.
cudaError_t launch_compress(const uint16_t* raw, const float* gate, const float* bias, int m,
                            const float* w_idx, int64_t T, int B, int64_t out_seq_stride,
                            uint8_t* kv_out, uint8_t* ikey_out, float* iscale_out, int num_sms,
                            cudaStream_t stream, int64_t pos0 = 0, double rope_base = 0.0, float kv_scale = 1.f,
                            bool perhead = false);
size_t compress_index_smem_bytes();
cudaError_t launch_compress_channel(const uint16_t* raw, const float* gate, const float* bias, int m,
                                    const float* w_idx, int64_t T, uint8_t* kv_out, uint8_t* ikey_out,
                                    float* iscale_out, int num_sms, cudaStream_t stream);

cudaError_t launch_prefill_state(const uint16_t* raw, const float* gate, int64_t T, int m, int W,
                                 int B, uint8_t* win_kv, uint16_t* tail_kv, float* tail_gate,
                                 int32_t* seq_len, cudaStream_t stream, double rope_base = 0.0,
                                 float kv_scale = 1.f);

cudaError_t launch_append(const csld_layer_cache& cache, const uint16_t* kv_new,
                          const float* gate_new, int32_t* err, cudaStream_t stream, double rope_base = 0.0,
                          float kv_scale = 1.f, bool perhead = false);

// Lightning indexer + top-k.
struct IndexerPlan {
    bool coop;          // one cooperative pass (all CTAs resident) instead of the merge tree
    int chunk;          // entries per scoring CTA (multiple of 256)
    int n_chunks;       // chunks (ranges) per sequence (over the capacity)
    int kc;             // candidates kept per chunk = min(k, chunk)
    int group;          // runs merged by one CTA in the merge tree
    bool levels_ok;     // the merge tree reaches one run within its level limit
    size_t ws_bytes;    // workspace bytes (must be zero-filled before first use)
};
IndexerPlan indexer_plan(int B, int64_t cap, int k, int num_sms);
cudaError_t launch_indexer(const uint8_t* ikeys, const float* iscales, int64_t cap,
                           const int32_t* seq_len, int ratio, const float* q_idx,
                           const float* head_w, int B, int k, int32_t* topk_out, void* ws,
                           const IndexerPlan& plan, int32_t* err, cudaStream_t stream);

// Test hook of the cooperative indexer (see csld_test_set_barrier_extra).
extern std::atomic<int> g_test_barrier_extra;

// Hybrid decode attention.
struct AttentionPlan {
    int splits;         // CTAs per sequence
    size_t ws_bytes;
};
AttentionPlan attention_plan(int B, int64_t cap, int k, bool sparse, int W, int num_sms);
// B cache rows with Q query rows each (query j of row b sees the first seq_len[b] - Q + 1 + j
// tokens); the window ring has Wr >= W slots per cache row.  The plan counts B * Q rows.
// kv_scale: the entries' FP8 dims stand for kv_scale times their code value (1: base layout).
cudaError_t launch_attention(const uint16_t* q, const uint8_t* comp_kv, int64_t cap, int ratio,
                             const int32_t* topk, int k, const uint8_t* win_kv, int W, int Wr, int Q,
                             const int32_t* seq_len, int B, float scale, float* out,
                             float* lse_out, void* ws, const AttentionPlan& plan, int32_t* err,
                             cudaStream_t stream, float kv_scale = 1.f);

// Device address of the library-owned attention scratch on the current device (looked up on
// the first call per device).
cudaError_t attention_static_scratch(void** ptr);
// The tensor-core (tcgen05) partial kernel of the hybrid decode attention (attention_tc.cu).
int attention_tc_tile();
size_t attention_tc_smem_bytes();
cudaError_t launch_attention_tc_partial(const uint16_t* q, const uint8_t* comp_kv, int64_t cap, int ratio,
                                        const int32_t* topk, int k, const uint8_t* win_kv, int W, int Wr, int Q,
                                        const int32_t* seq_len, int B, float scale, int splits, float* opart,
                                        float2* mlpart, int32_t* err, cudaStream_t stream, float kv_scale);

}  // namespace csld
