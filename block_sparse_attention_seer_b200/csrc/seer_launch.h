// seer_launch.h -- host-side launchers of the kernels behind the C ABI.
// Arguments are assumed validated by the caller (seer_api.cu).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace seer {

struct Shape {
    int B, Hq, Hkv, G, D, dg, blk, Lmax, NBmax;
};

cudaError_t launch_kpool_update(const Shape& s, const void* k_cache, const float* w_k, const int32_t* seq_lens,
                                const int32_t* upd_start, float* kpool, int num_sms, cudaStream_t stream);

cudaError_t launch_gate_scores(const Shape& s, const void* q, const float* w_q, const float* kpool,
                               const int32_t* seq_lens, float* scores, int num_sms, cudaStream_t stream);

cudaError_t launch_select_blocks(const Shape& s, const float* scores, const int32_t* seq_lens, int kmax,
                                 int32_t* block_idx, int32_t* num_selected, cudaStream_t stream);

struct DecodeLaunch {
    const void* q;
    const int32_t* seq_lens;
    const int32_t* block_idx;
    const int32_t* num_selected;
    float* o_part;
    float* lse_part;
    int kmax;
    int num_splits;
    float sm_scale;
};

// tmap_k / tmap_v: 2-D bf16 maps over [B*Hkv*Lmax rows, D cols], box 64 x blk,
// 128-byte swizzle (built by the caller).
cudaError_t launch_sparse_decode(const Shape& s, const DecodeLaunch& a, const CUtensorMap& tmap_k,
                                 const CUtensorMap& tmap_v, int num_sms, cudaStream_t stream);

// Number of CTAs the decode kernel runs for these arguments (1 per SM at most).
int sparse_decode_ctas(const Shape& s, int kmax, int num_splits, int num_sms);

// The whole decode step in one cooperative launch (sparse_decode.cu).
struct StepLaunch {
    const void* q;
    const void* k_cache;
    const void* v_cache;
    const float* w_q;
    const float* w_k;
    const int32_t* seq_lens;
    const int32_t* upd_start;  // NULL: refresh the last block only
    int budget_tokens;
    float sm_scale;  // resolved (> 0)
    float* kpool;
    int32_t* block_idx;
    int32_t* num_selected;
    void* out;
    float* lse_out;
    void* workspace;
};

// Byte offsets inside the step's workspace: the launch counter, the two
// tallies of fully taken rows, per-row gate counts and decode states (all
// zero before the first call: [0, counters_end)), then the gate's order keys
// and the decode's partial slots.
struct WorkspaceLayout {
    size_t launch_ctr, rows_taken, row_cnt, row_state, counters_end, keys, o_part, lse_part, total;
};
WorkspaceLayout step_workspace_layout(const Shape& s, int kmax, int num_sms);

cudaError_t launch_decode_step(const Shape& s, const StepLaunch& a, const CUtensorMap& tmK, const CUtensorMap& tmV,
                               int num_sms, cudaStream_t stream);

// The same step with its scratch in a static device array instead of a caller
// workspace (no allocation anywhere); static_scratch_bytes() is the array's size.
size_t static_scratch_bytes();
cudaError_t launch_decode_step_static(const Shape& s, StepLaunch a, const CUtensorMap& tmK, const CUtensorMap& tmV,
                                      int num_sms, cudaStream_t stream);

// Failure detection: the decode kernel's count of CTAs that gave up on a
// bounded wait, and a self-test of the bounded wait (synchronous).
cudaError_t read_decode_wait_failures(unsigned int* count, bool reset);
cudaError_t run_wait_selftest(unsigned long long limit_ns, int* timed_out);

// Gate variants (gate_variants.cu): per-head scores aggregated over the group
// (0 mean, 1 max, 2 mean of each head's softmax over its row's blocks), and
// threshold selection (at most kmax - 1 candidates scoring >= tau, plus the last block).
cudaError_t launch_gate_scores_agg(const Shape& s, const void* q, const float* w_q, const float* kpool,
                                   const int32_t* seq_lens, int agg, float* scores, int num_sms, cudaStream_t stream);
cudaError_t launch_select_threshold(const Shape& s, const float* scores, const int32_t* seq_lens, int kmax, float tau,
                                    int32_t* block_idx, int32_t* num_selected, cudaStream_t stream);

// Block-sparse prefill (prefill.cu): query-block gate scores [B, Hkv, NBmax, NBmax]
// (j <= i), per-query-block selection [B, Hkv, NBmax, kmax] / [B, Hkv, NBmax], and
// causal block-sparse attention out bf16 [B, Hq, Lmax, D], lse [B, Hq, Lmax] (nullable).
cudaError_t launch_prefill_gate(const Shape& s, const void* q, const float* w_q, const float* kpool,
                                const int32_t* seq_lens, float* scores, cudaStream_t stream);
cudaError_t launch_prefill_select(const Shape& s, const float* scores, const int32_t* seq_lens, int kmax,
                                  int32_t* block_idx, int32_t* num_selected, cudaStream_t stream);
// Attention (prefill_attn.cu, tcgen05): tmQ views q as [B*Hq*Lmax, D] with a
// 64-column x blk-row box, tmK / tmV view the caches as [B*Hkv*Lmax, D] with a
// 64 x 64 box; all 128-byte swizzled.
cudaError_t launch_prefill_attention(const Shape& s, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                                     const CUtensorMap& tmV, const int32_t* seq_lens, const int32_t* block_idx,
                                     const int32_t* num_selected, int kmax, float sm_scale, void* out, float* lse_out,
                                     cudaStream_t stream);

// Block-level ground truth: each query head's dense softmax mass per KV block
// [B, Hq, NBmax] and lse [B, Hq] (nullable) (block_mass.cu).
cudaError_t launch_block_mass(const Shape& s, const void* q, const void* k_cache, const int32_t* seq_lens,
                              float sm_scale, float* mass, float* lse_out, cudaStream_t stream);

// New token's K and V rows [B, Hkv, D] -> position L_b - 1 of the caches (append_kv.cu).
cudaError_t launch_append_kv(const Shape& s, const void* k_new, const void* v_new, const int32_t* seq_lens,
                             void* k_cache, void* v_cache, cudaStream_t stream);

cudaError_t launch_combine(const Shape& s, const float* o_part, const float* lse_part, int num_splits,
                           void* out, float* lse_out, cudaStream_t stream);

}  // namespace seer
