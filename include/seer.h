/*
 * seer.h -- C ABI of the B200 (sm_100a) gated block-sparse decode library.
 *
 * The library computes one decode step of SeerAttention-R's sparse attention
 * over a grouped-query (GQA) KV cache:
 *
 *   a1 seer_kpool_update   pooled-and-projected K per KV block (the gate's
 *                          key side, kept as a cache)
 *   a2 seer_gate_scores    one gating score per (batch, KV head, block) from
 *                          the un-pooled decode query
 *   a3 seer_select_blocks  the kept blocks under a token budget
 *   a4 seer_sparse_decode  split-KV flash-decode over the kept blocks only
 *   a5 seer_combine        merge of the split partials into the output
 * and, around them: seer_append_kv (the step's token into the caches),
 * seer_decode_step (a1..a5 as one launch) and seer_block_mass (the gate's
 * block-level ground truth).
 *
 * Sources: "SeerAttention-R: Sparse Attention Adaptation for Long Reasoning"
 * (abstract) for the decode setting, the un-pooled query, the token budget and
 * the 64/128 block sizes; "SeerAttention: Learning Intrinsic Sparse Attention
 * in Your LLMs" (abstract) for the gate itself (pool along the sequence,
 * learnable linear layers, multiply to get block scores).
 *
 * Conventions shared by every call:
 *  - All tensor arguments are DEVICE pointers to dense row-major arrays with
 *    the shapes given below. The caller allocates, owns and frees every
 *    buffer; the library never allocates, frees or synchronises, and keeps no
 *    state between calls.
 *  - `dims` is read during the call only. NBmax = ceil(max_seq_len /
 *    block_size) and G = num_q_heads / num_kv_heads.
 *  - bf16 arrays are passed as `const void*` (IEEE bfloat16, 2 bytes).
 *  - Work is enqueued on `stream` (NULL: the legacy default stream); calls
 *    return before it runs.
 *  - Arguments are validated on the host before anything is launched: a bad
 *    pointer or shape returns SEER_ERR_INVALID_ARG, an unsupported size
 *    SEER_ERR_UNSUPPORTED, and nothing is enqueued. A failed launch returns
 *    SEER_ERR_CUDA. Faults inside a kernel surface at the caller's next
 *    synchronisation, as for any CUDA kernel.
 *  - Values held in device memory (sequence lengths, block lists) cannot be
 *    checked on the host. A sequence length of 0 means an empty row (no block
 *    kept, output 0, lse -inf); lengths above max_seq_len are clamped to it;
 *    block indices outside [0, NB_b) are skipped by the decode kernel.
 *  - Supported sizes: head_dim in {64, 128}, gate_dim in {64, 128},
 *    block_size in {64, 128}, 1 <= G <= 8, num_q_heads % num_kv_heads == 0,
 *    max_seq_len <= 2^24, batch * num_kv_heads * max_seq_len < 2^31.
 */
#ifndef SEER_H_
#define SEER_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SEER_OK = 0,
    SEER_ERR_INVALID_ARG = 1,
    SEER_ERR_UNSUPPORTED = 2,
    SEER_ERR_CUDA = 3
} seer_status;

typedef struct {
    int32_t batch;        /* B */
    int32_t num_q_heads;  /* Hq */
    int32_t num_kv_heads; /* Hkv; G = Hq / Hkv query heads share one KV head */
    int32_t head_dim;     /* D */
    int32_t gate_dim;     /* dg, width of the gate's projected space */
    int32_t block_size;   /* blk, tokens per sparse-attention block */
    int32_t max_seq_len;  /* Lmax, tokens allocated per (b, kv head) in the caches */
} seer_dims;

/*
 * a1. Pooled-K cache update ("SeerAttention", abstract: the gate pools K along
 * the sequence dimension and passes it through a learnable linear layer).
 *
 * For every block j that holds a token in [upd_start[b], L_b), with
 * L_b = seq_lens[b] and n_j the number of its tokens below L_b:
 *     kpool[b,kvh,j,:] = W_k[kvh] . ( (1/n_j) * sum_{t in block j, t < L_b} K[b,kvh,t,:] )
 * Other blocks are left untouched. upd_start = NULL rebuilds every block
 * (after a prefill); upd_start[b] = L_b - 1 refreshes only the open last
 * block (a decode step). Pooling and projection accumulate in fp32.
 *
 *   k_cache   bf16 [B, Hkv, Lmax, D]
 *   w_k       fp32 [Hkv, dg, D]
 *   seq_lens  int32 [B]
 *   upd_start int32 [B] or NULL
 *   kpool     fp32 [B, Hkv, NBmax, dg]   (output)
 */
seer_status seer_kpool_update(const seer_dims* dims, const void* k_cache, const float* w_k,
                              const int32_t* seq_lens, const int32_t* upd_start, float* kpool,
                              cudaStream_t stream);

/*
 * a2. Gate scores ("SeerAttention-R", abstract: query pooling removed for
 * decoding, so the decode query is used as is; "SeerAttention", abstract: the
 * projected query and key are multiplied to give block scores).
 *
 *     s[b,kvh,j] = (1/G) sum_{h in group(kvh)} (W_q[kvh] . q[b,h,:]) . kpool[b,kvh,j,:] / sqrt(dg)
 * for j < NB_b = ceil(L_b / blk); entries j >= NB_b are not written.
 *
 *   q        bf16 [B, Hq, D]      (the decode query, one token per sequence)
 *   w_q      fp32 [Hkv, dg, D]
 *   kpool    fp32 [B, Hkv, NBmax, dg]
 *   seq_lens int32 [B]
 *   scores   fp32 [B, Hkv, NBmax]  (output)
 */
seer_status seer_gate_scores(const seer_dims* dims, const void* q, const float* w_q,
                             const float* kpool, const int32_t* seq_lens, float* scores,
                             cudaStream_t stream);

/*
 * a3. Block selection under a token budget ("SeerAttention-R", abstract: a
 * 4K-token budget at block sizes 64/128).
 *
 * kmax = budget_tokens / block_size, k_b = min(kmax, NB_b). Row (b, kvh)
 * keeps block NB_b - 1 (the open, possibly partial, last block) and the
 * k_b - 1 highest-scoring blocks among 0 .. NB_b - 2; equal scores are
 * broken toward the lower block index. The kept indices are written in
 * ascending order to block_idx[b,kvh,0..k_b-1], the remaining slots get -1,
 * and num_selected[b,kvh] = k_b.
 *
 *   scores        fp32 [B, Hkv, NBmax]
 *   seq_lens      int32 [B]
 *   budget_tokens a positive multiple of block_size
 *   block_idx     int32 [B, Hkv, kmax]  (output)
 *   num_selected  int32 [B, Hkv]        (output)
 * Errors: budget_tokens not a positive multiple of block_size, or
 * NBmax > 16384, give SEER_ERR_INVALID_ARG / SEER_ERR_UNSUPPORTED.
 */
seer_status seer_select_blocks(const seer_dims* dims, const float* scores, const int32_t* seq_lens,
                               int32_t budget_tokens, int32_t* block_idx, int32_t* num_selected,
                               cudaStream_t stream);

/*
 * a4. Block-sparse split-KV flash-decode ("SeerAttention-R", abstract: a
 * sparse decoding kernel that reads only the kept blocks).
 *
 * For each query head h of KV head kvh, softmax attention of q[b,h] over the
 * tokens t < L_b of the blocks listed in block_idx[b,kvh,0..num_selected-1]:
 *     z_t = sm_scale * q[b,h,:] . K[b,kvh,t,:],   out = sum_t softmax(z)_t V[b,kvh,t,:]
 * computed as partial results over disjoint pieces of the block list. Slot s
 * of (b, h) receives the normalised partial output o_part[b,h,s,:] and its
 * log-denominator lse_part[b,h,s] (natural log, scaled logits); a slot with
 * no tokens has lse_part = -inf and its o_part is not written. seer_combine
 * merges the slots.
 *
 * Scheduling: the kernel is persistent. The kept blocks of all rows, laid end
 * to end with kmax positions reserved per row, are cut into P equal ranges,
 * one per CTA; each (CTA, row) overlap is one slot. P is the device's SM
 * count when num_splits >= min(kmax, SMs), else num_splits, so that no row
 * ever needs more than num_splits slots. seer_default_num_splits() returns
 * min(kmax, SMs).
 *
 *   q            bf16 [B, Hq, D]
 *   k_cache      bf16 [B, Hkv, Lmax, D]
 *   v_cache      bf16 [B, Hkv, Lmax, D]
 *   seq_lens     int32 [B]
 *   block_idx    int32 [B, Hkv, kmax]   (any order; a dense decode passes 0..NB_b-1)
 *   num_selected int32 [B, Hkv]          (values above kmax are clamped to kmax)
 *   kmax         row stride of block_idx, >= 1
 *   num_splits   S, slots per (b, h), >= 1
 *   sm_scale     softmax scale; <= 0 selects 1/sqrt(D)
 *   o_part       fp32 [B, Hq, S, D]     (output)
 *   lse_part     fp32 [B, Hq, S]        (output)
 * The K/V caches must be 16-byte aligned (TMA); bf16 values only.
 */
seer_status seer_sparse_decode(const seer_dims* dims, const void* q, const void* k_cache,
                               const void* v_cache, const int32_t* seq_lens, const int32_t* block_idx,
                               const int32_t* num_selected, int32_t kmax, int32_t num_splits,
                               float sm_scale, float* o_part, float* lse_part, cudaStream_t stream);

/*
 * a5. Merge of the split partials (log-sum-exp weighted):
 *     M = max_s lse_s,  w_s = exp(lse_s - M),
 *     out = sum_s w_s o_s / sum_s w_s,  lse = M + log(sum_s w_s)
 * Slots with lse = -inf are skipped; if every slot is -inf, out = 0 and
 * lse = -inf.
 *
 *   o_part     fp32 [B, Hq, S, D]
 *   lse_part   fp32 [B, Hq, S]
 *   num_splits S, as passed to seer_sparse_decode
 *   out        bf16 [B, Hq, D]   (output)
 *   lse_out    fp32 [B, Hq]      (output, may be NULL)
 */
seer_status seer_combine(const seer_dims* dims, const float* o_part, const float* lse_part,
                         int32_t num_splits, void* out, float* lse_out, cudaStream_t stream);

/* Block-sparse prefill. "SeerAttention: Learning Intrinsic Sparse Attention
 * in Your LLMs" (abstract): pool Q and K along the sequence, pass them
 * through the learnable linear layers, multiply into block-level scores and
 * run a block-sparse attention over the kept blocks. Read for a causal prompt
 * of L_b tokens (L_b = clamped seq_lens[b]) with query and key blocks of
 * block_size tokens, the gate and selection readings of the decode path:
 *
 * seer_prefill_gate_scores:
 *   qbar[b, kvh, i] = mean over the group's heads and the valid tokens of
 *                     query block i of q[b, h, t, :]
 *   scores[b, kvh, i, j] = (W_q[kvh] qbar) . kpool[b, kvh, j] / sqrt(dg),
 *                     j <= i < NB_b; other entries are left undefined.
 *   q        bf16 [B, Hq, Lmax, D]  (16-byte aligned; token t of head h at [b, h, t, :])
 *   kpool    fp32 [B, Hkv, NBmax, dg]  (seer_kpool_update over the prompt)
 *   scores   fp32 [B, Hkv, NBmax, NBmax]
 *
 * seer_prefill_select_blocks: for each query block i < NB_b, block i itself
 * plus the top min(k, i + 1) - 1 of blocks 0 .. i-1 (higher score, then lower
 * index), ascending; k = budget_tokens / block_size. -1 fills the rest; query
 * blocks i >= NB_b get num_selected 0.
 *   block_idx     int32 [B, Hkv, NBmax, kmax]
 *   num_selected  int32 [B, Hkv, NBmax]
 *
 * seer_prefill_attention: token t < L_b of query block i = t / block_size,
 * head h: out = softmax(q_t . K_u * sm_scale) V_u over the tokens u <= t,
 * u < L_b, of the kept blocks of (b, kvh, i) (entries outside [0, i] are
 * skipped); lse its natural-log denominator. Rows t >= L_b: out 0, lse -inf.
 * sm_scale <= 0 means 1/sqrt(D). Runs on the tcgen05 tensor cores (bf16
 * products, fp32 accumulation; P rounded to bf16 for P V). A bounded wait that
 * gives up leaves NaN in the rows of the CTA concerned.
 *   q, k_cache, v_cache  16-byte aligned
 *   k_cache, v_cache  bf16 [B, Hkv, Lmax, D]
 *   out               bf16 [B, Hq, Lmax, D]  (output, 16-byte aligned)
 *   lse_out           fp32 [B, Hq, Lmax]     (output, may be NULL)
 *
 * Errors: SEER_ERR_INVALID_ARG for NULL/unaligned pointers, bad budgets or
 * scales; SEER_ERR_UNSUPPORTED when NBmax > 4096, batch x num_kv_heads > 65535,
 * batch x num_q_heads x max_seq_len >= 2^31 or outside the supported sizes.
 */
seer_status seer_prefill_gate_scores(const seer_dims* dims, const void* q, const float* w_q, const float* kpool,
                                     const int32_t* seq_lens, float* scores, cudaStream_t stream);
seer_status seer_prefill_select_blocks(const seer_dims* dims, const float* scores, const int32_t* seq_lens,
                                       int32_t budget_tokens, int32_t* block_idx, int32_t* num_selected,
                                       cudaStream_t stream);
seer_status seer_prefill_attention(const seer_dims* dims, const void* q, const void* k_cache, const void* v_cache,
                                   const int32_t* seq_lens, const int32_t* block_idx, const int32_t* num_selected,
                                   int32_t kmax, float sm_scale, void* out, float* lse_out, cudaStream_t stream);

/* Gate variants. Neither page says how the G query heads of a GQA group share
 * one block score, nor whether a threshold may replace the token budget; the
 * mean gate and top-k above are the plain readings, these are the
 * alternatives (every head scored on its own first):
 *   s_h[j] = (W_q q_h) . kpool[b, kvh, j] / sqrt(dg)
 *   SEER_AGG_MEAN          s[j] = (1/G) sum_h s_h[j]   (same as seer_gate_scores up to rounding)
 *   SEER_AGG_MAX           s[j] = max_h s_h[j]
 *   SEER_AGG_SOFTMAX_MEAN  s[j] = (1/G) sum_h exp(s_h[j]) / sum_{i < NB_b} exp(s_h[i])
 * Arguments, layouts and errors as seer_gate_scores; an aggregation outside
 * the three values is SEER_ERR_INVALID_ARG.
 *
 * seer_select_blocks_threshold keeps block NB_b - 1 plus the candidates
 * 0 .. NB_b - 2 whose score is >= threshold, at most k_b - 1 of them (the
 * highest; equal scores to the lower index), ascending; num_selected = their
 * count + 1 (0 for an empty sequence); -1 fills the rest of the kmax slots.
 * threshold = -inf gives seer_select_blocks. Arguments as seer_select_blocks;
 * a NaN threshold is SEER_ERR_INVALID_ARG.
 */
enum { SEER_AGG_MEAN = 0, SEER_AGG_MAX = 1, SEER_AGG_SOFTMAX_MEAN = 2 };
seer_status seer_gate_scores_agg(const seer_dims* dims, const void* q, const float* w_q, const float* kpool,
                                 const int32_t* seq_lens, int32_t aggregation, float* scores, cudaStream_t stream);
seer_status seer_select_blocks_threshold(const seer_dims* dims, const float* scores, const int32_t* seq_lens,
                                         int32_t budget_tokens, float threshold, int32_t* block_idx,
                                         int32_t* num_selected, cudaStream_t stream);

/* Block-level ground truth of one decode query. "SeerAttention: Learning
 * Intrinsic Sparse Attention in Your LLMs" (abstract) distils its gate from a
 * block-level ground truth extracted by a customised attention kernel; read
 * for a decode query it is the share of each query head's dense softmax that
 * falls in each KV block:
 *   z_t = sm_scale * q_h . K[b, kvh, t],  t < L_b (L_b = clamped seq_lens[b])
 *   mass[b, h, j] = sum_{t in block j} exp(z_t) / sum_t exp(z_t)   (j < NB_b)
 *   mass[b, h, j] = 0                                               (j >= NB_b)
 *   lse_out[b, h] = log sum_t exp(z_t)        (-inf when L_b = 0; mass all 0)
 * sm_scale <= 0 means 1/sqrt(head_dim). Two launches (per-block log-masses
 * into `mass`, then a per-row normalisation in place); reads all of K once.
 *
 *   q        bf16 [B, Hq, D]            (16-byte aligned)
 *   k_cache  bf16 [B, Hkv, Lmax, D]     (16-byte aligned)
 *   seq_lens int32 [B]
 *   mass     fp32 [B, Hq, NBmax]        (output)
 *   lse_out  fp32 [B, Hq]               (output, may be NULL)
 *
 * Errors: SEER_ERR_INVALID_ARG for NULL/unaligned pointers, a NaN or infinite
 * sm_scale or invalid dims; SEER_ERR_UNSUPPORTED outside the supported sizes.
 */
seer_status seer_block_mass(const seer_dims* dims, const void* q, const void* k_cache, const int32_t* seq_lens,
                            float sm_scale, float* mass, float* lse_out, cudaStream_t stream);

/* Appending the step's token. "SeerAttention-R" (abstract) decodes
 * auto-regressively: each step appends one token whose K and V take part in
 * that same step. seer_append_kv writes the token's rows at position
 * L_b - 1 of every (b, kv head) row of both caches (L_b = clamped
 * seq_lens[b], the length AFTER the append; rows with L_b = 0 are left
 * alone), so a caller ships q and the new K/V per step and no strided cache
 * slices. Call it before the step on the same stream. No counterpart on the
 * pages beyond the decode setting itself.
 *
 *   k_new, v_new  bf16 [B, Hkv, D]        (16-byte aligned)
 *   seq_lens      int32 [B]
 *   k_cache       bf16 [B, Hkv, Lmax, D]  (written at [b, kvh, L_b - 1, :])
 *   v_cache       bf16 [B, Hkv, Lmax, D]  (idem)
 *
 * Errors: SEER_ERR_INVALID_ARG for NULL or unaligned pointers and invalid
 * dims; SEER_ERR_UNSUPPORTED for head_dim outside {64, 128}.
 */
seer_status seer_append_kv(const seer_dims* dims, const void* k_new, const void* v_new, const int32_t* seq_lens,
                           void* k_cache, void* v_cache, cudaStream_t stream);

/*
 * The whole decode step, a1..a5, in ONE cooperative launch (one CTA per SM),
 * with no grid-wide barrier. The gate spreads the pooled-key positions of the
 * (b, kvh) rows over the CTAs: it refreshes kpool for the blocks touching
 * [upd_start[b], L_b) (NULL: the last block only, i.e. the token just
 * appended), scores every other block with the same arithmetic as
 * seer_gate_scores and selects as seer_select_blocks does (bit-identical
 * block lists); the CTA that completes a row's gate publishes the row (a
 * release flag). The decode of a row starts as soon as it is published: when
 * rows fit the grid, the CTAs that gated a row stream even, fixed parts of its
 * kept list (a row held by one CTA is written straight to out, and its first
 * blocks, those the selection keeps whatever the rest of its search finds,
 * start streaming before the list is complete); when rows
 * outnumber the CTAs, CTAs take pieces of each list from the front and help
 * with the rows that have most left from the back. The CTA that completes a
 * row's positions merges its partial results into out / lse_out as
 * seer_combine does. One launch, no host synchronisation.
 * (The step of "SeerAttention-R: Sparse Attention Adaptation for Long
 * Reasoning", abstract; gate of "SeerAttention: Learning Intrinsic Sparse
 * Attention in Your LLMs", abstract.)
 *
 *   q, k_cache, v_cache, w_q, w_k, seq_lens   as above
 *   upd_start     int32 [B] or NULL (NULL: L_b - 1)
 *   budget_tokens a positive multiple of block_size; kmax = budget_tokens / block_size
 *   sm_scale      <= 0 selects 1/sqrt(D)
 *   kpool         fp32 [B, Hkv, NBmax, dg], read, and written for refreshed blocks
 *   block_idx     int32 [B, Hkv, kmax] (output: the kept blocks, as seer_select_blocks)
 *   num_selected  int32 [B, Hkv]       (output)
 *   out           bf16 [B, Hq, D]      (output)
 *   lse_out       fp32 [B, Hq]         (output, may be NULL)
 *   workspace     device scratch of at least seer_decode_step_workspace_size()
 *                 bytes, 256-byte aligned, ZERO-FILLED before its first use on a
 *                 device; every call leaves it ready for the next one (each
 *                 launch takes the next epoch from a counter in it and tags
 *                 what it publishes with that epoch; re-zero it after a call
 *                 that reported a wait failure). Use one workspace with one
 *                 device only. Calls that share a workspace must not overlap
 *                 on the GPU.
 * Repeatability: block_idx, num_selected and kpool are the same bit for bit on
 * every call with the same inputs. With no more (b, kvh) rows than SMs, out and
 * lse_out are too (fixed parts merged in a fixed order); with more rows, the
 * split of a row among CTAs depends on timing and out / lse_out may differ
 * between calls by the rounding of the fp32 merge (a bf16 unit in the last
 * place at most, in practice).
 * Errors: as the separate calls; SEER_ERR_CUDA also when the cooperative launch
 * cannot place one CTA on every SM (e.g. the device is shared with other work).
 */
seer_status seer_decode_step_workspace_size(const seer_dims* dims, int32_t budget_tokens, size_t* bytes);

seer_status seer_decode_step(const seer_dims* dims, const void* q, const void* k_cache, const void* v_cache,
                             const float* w_q, const float* w_k, const int32_t* seq_lens, const int32_t* upd_start,
                             int32_t budget_tokens, float sm_scale, float* kpool, int32_t* block_idx,
                             int32_t* num_selected, void* out, float* lse_out, void* workspace,
                             size_t workspace_bytes, cudaStream_t stream);

/*
 * seer_decode_step without a workspace argument, for callers that cannot
 * allocate device memory: e.g. a plugin whose host framework passes it only
 * its input and output tensors, or a serving loop that may not call
 * cudaMalloc (which can synchronise the whole device) once it is running.
 * (No counterpart in the papers: an interface convenience.)
 *
 * The scratch lives in a static device array of 32 MiB inside the library:
 * every GPU that loads the library holds one copy until the process exits.
 * Sizes whose scratch (seer_decode_step_workspace_size) exceeds 32 MiB are
 * rejected with SEER_ERR_UNSUPPORTED (seer_last_error_string says why); use
 * seer_decode_step for them. Nothing is allocated or freed: the first call
 * on a device looks up the array's device address (cudaGetSymbolAddress)
 * with that device current, so make that first call before any stream
 * capture; each call then clears the array's counters (an async memset on
 * `stream`) and launches the same kernel as seer_decode_step.
 * Every call on a device shares the one array: calls whose executions
 * overlap on the GPU (different streams, no ordering between them) race.
 * Arguments, outputs and errors otherwise as seer_decode_step.
 */
seer_status seer_decode_step_noalloc(const seer_dims* dims, const void* q, const void* k_cache, const void* v_cache,
                                     const float* w_q, const float* w_k, const int32_t* seq_lens,
                                     const int32_t* upd_start, int32_t budget_tokens, float sm_scale, float* kpool,
                                     int32_t* block_idx, int32_t* num_selected, void* out, float* lse_out,
                                     cudaStream_t stream);

/*
 * Slots per (b, h) that let seer_sparse_decode use every SM of the current
 * device: min(kmax, number of SMs). Host-only query (no launch).
 */
seer_status seer_default_num_splits(int32_t kmax, int32_t* num_splits);

/*
 * Failure detection (no page counterpart). Every wait inside the decode kernel
 * is bounded (1 s); a CTA that gives up writes NaN into the slot it was
 * producing (so the combined output is NaN) and increments a device counter.
 *
 * seer_decode_wait_failures: *count = that counter for the current device
 * (0 in normal operation); reset != 0 clears it. Synchronous: it waits for
 * work already queued on the legacy default stream.
 */
seer_status seer_decode_wait_failures(uint32_t* count, int32_t reset);

/*
 * Self-test of the bounded wait: one CTA waits, for at most limit_ns
 * (0 .. 2e9), on an mbarrier that nothing arrives at. *timed_out = 1 when the
 * wait gave up as designed (0 if it completed, which would be a fault of the
 * wait). The device stays usable afterwards. Synchronous (device-wide sync).
 */
seer_status seer_wait_selftest(int64_t limit_ns, int32_t* timed_out);

/* The CUDA error behind the last SEER_ERR_CUDA returned on the calling host
 * thread ("name: description"), or "no error". Valid until the next call. */
const char* seer_last_error_string(void);

/* A short static description of a status code. */
const char* seer_status_string(seer_status status);

#ifdef __cplusplus
}
#endif

#endif /* SEER_H_ */
