/*
 * seer_oracle.c -- plain, slow fp64 CPU oracle of gated block-sparse decode
 * attention (the decode hot path of SeerAttention-R).
 *
 * TEST INFRASTRUCTURE. Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg load this library. The CUDA library never
 * calls it, and the two share no code: no kernels, headers, helpers or
 * constants. Every input arrives as the exact bits the GPU receives (bf16 as
 * raw 16-bit words, fp32 weights) and is widened here, exactly, to double.
 *
 * Sources of what is computed:
 *  [R]  "SeerAttention-R: Sparse Attention Adaptation for Long Reasoning",
 *       abstract: the self-distilled gate of SeerAttention is kept, query
 *       pooling is removed so that a single decode query can be gated; the
 *       gate is a plug-in beside frozen weights; a 4K-token budget at sparse
 *       block sizes 64/128; a sparse decoding kernel reads only kept blocks.
 *  [V1] "SeerAttention: Learning Intrinsic Sparse Attention in Your LLMs",
 *       abstract: the gate pools Q and K along the sequence dimension, passes
 *       them through learnable linear layers and multiplies the two results
 *       to obtain block-level gating scores.
 *
 * Readings taken where the pages are silent (each one is also listed in the
 * design notes of the repository):
 *  - pooling operator: arithmetic mean over the valid tokens of a block; the
 *    partial last block is averaged over its own token count;
 *  - linear layers: one bias-free map per KV head, W_k, W_q : [dg, D];
 *  - GQA: one score per (KV head, block), the mean over the G query heads of
 *    the group of their per-head scores;
 *  - score scale 1/sqrt(dg); no softmax over blocks (it would not change the
 *    ranking);
 *  - selection: the last (possibly partial) block is always kept and counts
 *    toward the budget; the other k_b - 1 are the top scores, ties broken by
 *    the lower block index; the list is returned in ascending order;
 *  - attention: softmax(q.K / sqrt(D)) over the valid tokens of the kept
 *    blocks; lse is the natural log of the softmax denominator (with the
 *    scaled logits).
 *
 * Parallelism: OpenMP over independent (batch, KV head) rows. Each row is
 * computed by one thread in a fixed order, so results do not depend on the
 * thread count.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int32_t batch, num_q_heads, num_kv_heads, head_dim, gate_dim, block_size, max_seq_len;
} oracle_dims;

/* Exact widening of a bfloat16 bit pattern: a bf16 value is the top half of
 * the fp32 value with the same bits. */
static double bf16_to_double(uint16_t h) {
    union { uint32_t u; float f; } x;
    x.u = ((uint32_t)h) << 16;
    return (double)x.f;
}

static int num_blocks(int len, int blk) { return (len + blk - 1) / blk; }

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Step 1 and 2 of the gate, [V1]: pool K over the tokens of each block, then
 * the linear layer W_k.
 *   pooled[j] = (1/n_j) sum_{t in block j, t < L_b} K[b,kvh,t,:]
 *   kpool[b,kvh,j,e] = sum_d W_k[kvh,e,d] * pooled[j,d]
 * Blocks j >= NB_b are filled with NaN (undefined). */
void oracle_pool_project(const oracle_dims* dm, const uint16_t* k_cache, const float* w_k,
                         const int32_t* seq_lens, double* kpool) {
    const int B = dm->batch, Hkv = dm->num_kv_heads, D = dm->head_dim, dg = dm->gate_dim;
    const int blk = dm->block_size, Lmax = dm->max_seq_len;
    const int NBmax = num_blocks(Lmax, blk);
#pragma omp parallel for schedule(dynamic, 1)
    for (int row = 0; row < B * Hkv; ++row) {
        const int b = row / Hkv, kvh = row % Hkv;
        const int L = seq_lens[b];
        const int NB = num_blocks(L, blk);
        double* pooled = (double*)malloc(sizeof(double) * (size_t)D);
        for (int j = 0; j < NBmax; ++j) {
            double* out = kpool + ((size_t)row * NBmax + j) * dg;
            if (j >= NB) {
                for (int e = 0; e < dg; ++e) out[e] = NAN;
                continue;
            }
            const int t0 = j * blk;
            const int t1 = (t0 + blk < L) ? t0 + blk : L;
            const int n = t1 - t0;
            for (int d = 0; d < D; ++d) pooled[d] = 0.0;
            for (int t = t0; t < t1; ++t) {
                const uint16_t* kt = k_cache + ((size_t)row * Lmax + t) * D;
                for (int d = 0; d < D; ++d) pooled[d] += bf16_to_double(kt[d]);
            }
            for (int d = 0; d < D; ++d) pooled[d] /= (double)n;
            const float* W = w_k + (size_t)kvh * dg * D;
            for (int e = 0; e < dg; ++e) {
                double acc = 0.0;
                for (int d = 0; d < D; ++d) acc += (double)W[(size_t)e * D + d] * pooled[d];
                out[e] = acc;
            }
        }
        free(pooled);
    }
}

/* Steps 3 and 4, [R] + [V1]: the un-pooled decode query of each head goes
 * through W_q, is multiplied with every pooled-K row, scaled by 1/sqrt(dg),
 * and the G heads of the group are averaged.
 *   qg[h,e]     = sum_d W_q[kvh,e,d] * q[b,h,d]
 *   s_h[j]      = sum_e qg[h,e] * kpool[b,kvh,j,e] / sqrt(dg)
 *   s[b,kvh,j]  = (1/G) sum_{h in group(kvh)} s_h[j]        for j < NB_b
 * Entries j >= NB_b are NaN. */
void oracle_gate_scores(const oracle_dims* dm, const uint16_t* q, const float* w_q,
                        const double* kpool, const int32_t* seq_lens, double* scores) {
    const int B = dm->batch, Hq = dm->num_q_heads, Hkv = dm->num_kv_heads;
    const int D = dm->head_dim, dg = dm->gate_dim, blk = dm->block_size;
    const int G = Hq / Hkv;
    const int NBmax = num_blocks(dm->max_seq_len, blk);
#pragma omp parallel for schedule(dynamic, 1)
    for (int row = 0; row < B * Hkv; ++row) {
        const int b = row / Hkv, kvh = row % Hkv;
        const int NB = num_blocks(seq_lens[b], blk);
        double* qg = (double*)malloc(sizeof(double) * (size_t)G * dg);
        const float* W = w_q + (size_t)kvh * dg * D;
        for (int h = 0; h < G; ++h) {
            const uint16_t* qh = q + ((size_t)b * Hq + (size_t)kvh * G + h) * D;
            for (int e = 0; e < dg; ++e) {
                double acc = 0.0;
                for (int d = 0; d < D; ++d) acc += (double)W[(size_t)e * D + d] * bf16_to_double(qh[d]);
                qg[(size_t)h * dg + e] = acc;
            }
        }
        const double inv_sqrt_dg = 1.0 / sqrt((double)dg);
        for (int j = 0; j < NBmax; ++j) {
            double* out = scores + (size_t)row * NBmax + j;
            if (j >= NB) { *out = NAN; continue; }
            const double* kp = kpool + ((size_t)row * NBmax + j) * dg;
            double s = 0.0;
            for (int h = 0; h < G; ++h) {
                double sh = 0.0;
                for (int e = 0; e < dg; ++e) sh += qg[(size_t)h * dg + e] * kp[e];
                s += sh * inv_sqrt_dg;
            }
            *out = s / (double)G;
        }
        free(qg);
    }
}

typedef struct { double score; int32_t index; } scored_block;

/* Higher score first; equal scores: lower block index first. */
static int by_score_then_index(const void* pa, const void* pb) {
    const scored_block* a = (const scored_block*)pa;
    const scored_block* b = (const scored_block*)pb;
    if (a->score > b->score) return -1;
    if (a->score < b->score) return 1;
    return (a->index < b->index) ? -1 : (a->index > b->index);
}

static int ascending_int(const void* pa, const void* pb) {
    const int32_t a = *(const int32_t*)pa, b = *(const int32_t*)pb;
    return (a > b) - (a < b);
}

/* Step 5, [R]: keep blocks within the token budget. k = budget/blk blocks,
 * k_b = min(k, NB_b). The last block NB_b-1 is always kept; the other
 * k_b-1 are the highest-scoring of blocks 0..NB_b-2 (ties: lower index).
 * Output: ascending indices in block_idx[b,kvh,0..k_b-1]; slots beyond k_b
 * are set to -1; num_selected[b,kvh] = k_b. */
void oracle_select(const oracle_dims* dm, const double* scores, const int32_t* seq_lens,
                   int32_t budget_tokens, int32_t* block_idx, int32_t* num_selected) {
    const int B = dm->batch, Hkv = dm->num_kv_heads, blk = dm->block_size;
    const int NBmax = num_blocks(dm->max_seq_len, blk);
    const int kmax = budget_tokens / blk;
#pragma omp parallel for schedule(dynamic, 1)
    for (int row = 0; row < B * Hkv; ++row) {
        const int b = row / Hkv;
        const int NB = num_blocks(seq_lens[b], blk);
        const int kb = (kmax < NB) ? kmax : NB;
        int32_t* out = block_idx + (size_t)row * kmax;
        const double* s = scores + (size_t)row * NBmax;
        if (NB == 0) { /* empty sequence: nothing to keep */
            for (int i = 0; i < kmax; ++i) out[i] = -1;
            num_selected[row] = 0;
            continue;
        }
        scored_block* cand = (scored_block*)malloc(sizeof(scored_block) * (size_t)(NB > 1 ? NB - 1 : 1));
        for (int j = 0; j < NB - 1; ++j) { cand[j].score = s[j]; cand[j].index = j; }
        qsort(cand, (size_t)(NB - 1), sizeof(scored_block), by_score_then_index);
        int n = 0;
        for (int i = 0; i < kb - 1; ++i) out[n++] = cand[i].index;
        out[n++] = NB - 1;
        qsort(out, (size_t)n, sizeof(int32_t), ascending_int);
        for (int i = n; i < kmax; ++i) out[i] = -1;
        num_selected[row] = n;
        free(cand);
    }
}

/* Step 6, [R]: softmax attention of each query head over the valid tokens of
 * the kept blocks of its KV head (the mask of a block-sparse decode):
 *   z_t = (q_h . K_t) * sm_scale, t in kept blocks, t < L_b
 *   out_h = sum_t softmax(z)_t V_t,   lse_h = log sum_t exp(z_t)
 * block_idx rows hold num_selected[b,kvh] entries (stride kmax); entries
 * outside [0, NB_b) are skipped. A row with no valid token gives out = 0 and
 * lse = -inf. sm_scale <= 0 means 1/sqrt(D). */
void oracle_attend(const oracle_dims* dm, const uint16_t* q, const uint16_t* k_cache,
                   const uint16_t* v_cache, const int32_t* seq_lens, const int32_t* block_idx,
                   const int32_t* num_selected, int32_t kmax, double sm_scale,
                   double* out, double* lse) {
    const int B = dm->batch, Hq = dm->num_q_heads, Hkv = dm->num_kv_heads;
    const int D = dm->head_dim, blk = dm->block_size, Lmax = dm->max_seq_len;
    const int G = Hq / Hkv;
    const double scale = (sm_scale > 0.0) ? sm_scale : 1.0 / sqrt((double)D);
#pragma omp parallel for schedule(dynamic, 1)
    for (int row = 0; row < B * Hkv; ++row) {
        const int b = row / Hkv, kvh = row % Hkv;
        const int L = seq_lens[b];
        const int NB = num_blocks(L, blk);
        const int32_t* idx = block_idx + (size_t)row * kmax;
        const int nsel = num_selected[row];
        /* token list of the kept blocks, in list order */
        int ntok = 0;
        for (int i = 0; i < nsel; ++i) {
            const int j = idx[i];
            if (j < 0 || j >= NB) continue;
            const int t1 = (j * blk + blk < L) ? j * blk + blk : L;
            ntok += t1 - j * blk;
        }
        double* z = (double*)malloc(sizeof(double) * (size_t)(ntok > 0 ? ntok : 1));
        int32_t* tok = (int32_t*)malloc(sizeof(int32_t) * (size_t)(ntok > 0 ? ntok : 1));
        int n = 0;
        for (int i = 0; i < nsel; ++i) {
            const int j = idx[i];
            if (j < 0 || j >= NB) continue;
            const int t1 = (j * blk + blk < L) ? j * blk + blk : L;
            for (int t = j * blk; t < t1; ++t) tok[n++] = t;
        }
        for (int h = 0; h < G; ++h) {
            const int hq = kvh * G + h;
            const uint16_t* qh = q + ((size_t)b * Hq + hq) * D;
            double* o = out + ((size_t)b * Hq + hq) * D;
            for (int d = 0; d < D; ++d) o[d] = 0.0;
            if (ntok == 0) { lse[(size_t)b * Hq + hq] = -INFINITY; continue; }
            double m = -INFINITY;
            for (int i = 0; i < ntok; ++i) {
                const uint16_t* kt = k_cache + ((size_t)row * Lmax + tok[i]) * D;
                double acc = 0.0;
                for (int d = 0; d < D; ++d) acc += bf16_to_double(qh[d]) * bf16_to_double(kt[d]);
                z[i] = acc * scale;
                if (z[i] > m) m = z[i];
            }
            double denom = 0.0;
            for (int i = 0; i < ntok; ++i) {
                const double p = exp(z[i] - m);
                denom += p;
                const uint16_t* vt = v_cache + ((size_t)row * Lmax + tok[i]) * D;
                for (int d = 0; d < D; ++d) o[d] += p * bf16_to_double(vt[d]);
            }
            for (int d = 0; d < D; ++d) o[d] /= denom;
            lse[(size_t)b * Hq + hq] = m + log(denom);
        }
        free(z);
        free(tok);
    }
}

/* Merge of partial softmax results over disjoint token sets: each part holds
 * the normalised output o_s and log-denominator lse_s of its own tokens.
 *   M = max_s lse_s,  w_s = exp(lse_s - M)
 *   out = sum_s w_s o_s / sum_s w_s,   lse = M + log sum_s w_s
 * Parts with lse = -inf carry no token and get weight 0. If every part is
 * empty, out = 0 and lse = -inf. Shapes: o_parts [n_parts, D], lse_parts
 * [n_parts]. */
void oracle_merge(int32_t n_parts, int32_t D, const double* o_parts, const double* lse_parts,
                  double* out, double* lse) {
    double M = -INFINITY;
    for (int s = 0; s < n_parts; ++s)
        if (lse_parts[s] > M) M = lse_parts[s];
    for (int d = 0; d < D; ++d) out[d] = 0.0;
    if (M == -INFINITY) { *lse = -INFINITY; return; }
    double wsum = 0.0;
    for (int s = 0; s < n_parts; ++s) {
        if (lse_parts[s] == -INFINITY) continue;
        const double w = exp(lse_parts[s] - M);
        wsum += w;
        for (int d = 0; d < D; ++d) out[d] += w * o_parts[(size_t)s * D + d];
    }
    for (int d = 0; d < D; ++d) out[d] /= wsum;
    *lse = M + log(wsum);
}

/* Block-level ground truth, [V1] (the customised attention that extracts the
 * block-level target the gate is distilled from) read for one decode query:
 * the dense softmax attention of each query head over all valid tokens, and
 * the share of its probability that falls in each block.
 *   z_t       = scale * q_h . K[b,kvh,t]            t < L_b (L_b clamped to [0, Lmax])
 *   p_t       = exp(z_t) / sum_{t'} exp(z_t')
 *   mass[j]   = sum_{t in block j, t < L_b} p_t      j < NB_b;  0 for j >= NB_b
 *   lse       = log sum_t exp(z_t)                   (-inf when L_b = 0)
 * Shapes: mass [B, Hq, NBmax], lse [B, Hq]. sm_scale <= 0 means 1/sqrt(D). */
void oracle_block_mass(const oracle_dims* dm, const uint16_t* q, const uint16_t* k_cache,
                       const int32_t* seq_lens, double sm_scale, double* mass, double* lse) {
    const int B = dm->batch, Hq = dm->num_q_heads, Hkv = dm->num_kv_heads;
    const int D = dm->head_dim, blk = dm->block_size, Lmax = dm->max_seq_len;
    const int G = Hq / Hkv;
    const int NBmax = num_blocks(Lmax, blk);
    const double scale = (sm_scale > 0.0) ? sm_scale : 1.0 / sqrt((double)D);
#pragma omp parallel for schedule(dynamic, 1)
    for (int row = 0; row < B * Hkv; ++row) {
        const int b = row / Hkv, kvh = row % Hkv;
        int L = seq_lens[b];
        L = L < 0 ? 0 : (L > Lmax ? Lmax : L);
        double* z = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
        for (int h = 0; h < G; ++h) {
            const int hq = kvh * G + h;
            const uint16_t* qh = q + ((size_t)b * Hq + hq) * D;
            double* mh = mass + ((size_t)b * Hq + hq) * NBmax;
            for (int j = 0; j < NBmax; ++j) mh[j] = 0.0;
            if (L == 0) { lse[(size_t)b * Hq + hq] = -INFINITY; continue; }
            double m = -INFINITY;
            for (int t = 0; t < L; ++t) {
                const uint16_t* kt = k_cache + ((size_t)row * Lmax + t) * D;
                double acc = 0.0;
                for (int d = 0; d < D; ++d) acc += bf16_to_double(qh[d]) * bf16_to_double(kt[d]);
                z[t] = acc * scale;
                if (z[t] > m) m = z[t];
            }
            double denom = 0.0;
            for (int t = 0; t < L; ++t) denom += exp(z[t] - m);
            for (int t = 0; t < L; ++t) mh[t / blk] += exp(z[t] - m) / denom;
            const double lse_h = m + log(denom);
            lse[(size_t)b * Hq + hq] = lse_h;
        }
        free(z);
    }
}

/* Gate variants (neither is on the pages; these are the readings taken).
 * Aggregation of the G per-head scores of a group, every head scored
 * explicitly (no use of linearity):
 *   s_h[j] = (W_q[kvh] q_h) . kpool[b,kvh,j] / sqrt(dg),  j < NB_b
 *   agg 0: s[j] = (1/G) sum_h s_h[j]                        (the mean gate)
 *   agg 1: s[j] = max_h s_h[j]
 *   agg 2: s[j] = (1/G) sum_h exp(s_h[j]) / sum_{i < NB_b} exp(s_h[i])
 *          (each head's softmax over all of its row's blocks, then the mean)
 * Entries j >= NB_b are NaN. */
void oracle_gate_scores_agg(const oracle_dims* dm, const uint16_t* q, const float* w_q,
                            const double* kpool, const int32_t* seq_lens, int32_t agg, double* scores) {
    const int B = dm->batch, Hq = dm->num_q_heads, Hkv = dm->num_kv_heads;
    const int D = dm->head_dim, dg = dm->gate_dim, blk = dm->block_size;
    const int NBmax = num_blocks(dm->max_seq_len, blk);
    const int G = Hq / Hkv;
    const double inv_sqrt_dg = 1.0 / sqrt((double)dg);
#pragma omp parallel for schedule(dynamic, 1)
    for (int row = 0; row < B * Hkv; ++row) {
        const int b = row / Hkv, kvh = row % Hkv;
        const int NB = num_blocks(seq_lens[b], blk);
        const float* W = w_q + (size_t)kvh * dg * D;
        double* qg = (double*)malloc(sizeof(double) * (size_t)G * dg);
        double* sh = (double*)malloc(sizeof(double) * (size_t)G * (NB > 0 ? NB : 1));
        for (int h = 0; h < G; ++h) {
            const uint16_t* qh = q + ((size_t)b * Hq + (size_t)kvh * G + h) * D;
            for (int e = 0; e < dg; ++e) {
                double acc = 0.0;
                for (int d = 0; d < D; ++d) acc += bf16_to_double(qh[d]) * (double)W[(size_t)e * D + d];
                qg[(size_t)h * dg + e] = acc;
            }
            for (int j = 0; j < NB; ++j) {
                const double* kp = kpool + (size_t)row * NBmax * dg + (size_t)j * dg;
                double acc = 0.0;
                for (int e = 0; e < dg; ++e) acc += qg[(size_t)h * dg + e] * kp[e];
                sh[(size_t)h * NB + j] = acc * inv_sqrt_dg;
            }
            if (agg == 2 && NB > 0) {  /* this head's softmax over its row's blocks */
                double m = -INFINITY, den = 0.0;
                for (int j = 0; j < NB; ++j) if (sh[(size_t)h * NB + j] > m) m = sh[(size_t)h * NB + j];
                for (int j = 0; j < NB; ++j) den += exp(sh[(size_t)h * NB + j] - m);
                for (int j = 0; j < NB; ++j) sh[(size_t)h * NB + j] = exp(sh[(size_t)h * NB + j] - m) / den;
            }
        }
        double* out = scores + (size_t)row * NBmax;
        for (int j = 0; j < NBmax; ++j) out[j] = NAN;
        for (int j = 0; j < NB; ++j) {
            double a = (agg == 1) ? -INFINITY : 0.0;
            for (int h = 0; h < G; ++h) {
                const double v = sh[(size_t)h * NB + j];
                if (agg == 1) a = v > a ? v : a;
                else a += v;
            }
            out[j] = (agg == 1) ? a : a / (double)G;
        }
        free(qg);
        free(sh);
    }
}

/* Threshold selection (a reading; the pages describe a token budget only):
 * block NB_b-1 always, plus the candidates 0 .. NB_b-2 whose score is at
 * least `threshold`, at most k_b - 1 of them (the highest, equal scores to the
 * lower index), ascending; -1 fills the rest of the kmax slots. */
void oracle_select_threshold(const oracle_dims* dm, const double* scores, const int32_t* seq_lens,
                             int32_t budget_tokens, double threshold, int32_t* block_idx,
                             int32_t* num_selected) {
    const int B = dm->batch, Hkv = dm->num_kv_heads, blk = dm->block_size;
    const int NBmax = num_blocks(dm->max_seq_len, blk);
    const int kmax = budget_tokens / blk;
    for (int row = 0; row < B * Hkv; ++row) {
        const int b = row / Hkv;
        const int NB = num_blocks(seq_lens[b], blk);
        const double* s = scores + (size_t)row * NBmax;
        int32_t* out = block_idx + (size_t)row * kmax;
        for (int i = 0; i < kmax; ++i) out[i] = -1;
        if (NB == 0) { num_selected[row] = 0; continue; }
        const int kb = kmax < NB ? kmax : NB;
        scored_block* cand = (scored_block*)malloc(sizeof(scored_block) * (size_t)NB);
        int nc = 0;
        for (int j = 0; j < NB - 1; ++j)
            if (s[j] >= threshold) { cand[nc].score = s[j]; cand[nc].index = j; ++nc; }
        qsort(cand, (size_t)nc, sizeof(scored_block), by_score_then_index);
        const int take = nc < kb - 1 ? nc : kb - 1;
        int n = 0;
        for (int i = 0; i < take; ++i) out[n++] = cand[i].index;
        qsort(out, (size_t)n, sizeof(int32_t), ascending_int);
        out[n] = NB - 1;
        num_selected[row] = n + 1;
        free(cand);
    }
}

/* ------------------------------------------------------------ block-sparse prefill
 * [V1] (pool Q and K along the sequence, linear layers, multiply to block
 * scores; a block-sparse attention over the kept blocks) read for a causal
 * prompt of L_b tokens, with the decode gate's readings (mean pool over valid
 * tokens, one bias-free map per KV head, mean over the group's heads, 1/sqrt(dg))
 * and selection rule (the diagonal block plays the decode's last block).
 * q: bf16 bits [B, Hq, Lmax, D]; query block i = tokens [i*blk, min((i+1)*blk, L_b)).
 *
 * Gate: qbar[h,i] = mean_{t in block i} q[b,h,t,:];  qg = W_q[kvh] qbar
 *   s[b,kvh,i,j] = (1/G) sum_h qg[h,i] . kpool[b,kvh,j] / sqrt(dg)   j <= i < NB_b
 * Entries with j > i or i >= NB_b are NaN. Shape [B, Hkv, NBmax, NBmax]. */
void oracle_prefill_gate(const oracle_dims* dm, const uint16_t* q, const float* w_q, const double* kpool,
                         const int32_t* seq_lens, double* scores) {
    const int B = dm->batch, Hq = dm->num_q_heads, Hkv = dm->num_kv_heads;
    const int D = dm->head_dim, dg = dm->gate_dim, blk = dm->block_size, Lmax = dm->max_seq_len;
    const int NBmax = num_blocks(Lmax, blk);
    const int G = Hq / Hkv;
    const double inv_sqrt_dg = 1.0 / sqrt((double)dg);
#pragma omp parallel for schedule(dynamic, 1)
    for (int row = 0; row < B * Hkv; ++row) {
        const int b = row / Hkv, kvh = row % Hkv;
        const int L = seq_lens[b];
        const int NB = num_blocks(L, blk);
        const float* W = w_q + (size_t)kvh * dg * D;
        double* qbar = (double*)malloc(sizeof(double) * (size_t)D);
        double* qg = (double*)malloc(sizeof(double) * (size_t)dg);
        double* out = scores + (size_t)row * NBmax * NBmax;
        for (size_t x = 0; x < (size_t)NBmax * NBmax; ++x) out[x] = NAN;
        for (int i = 0; i < NB; ++i) {
            const int t0 = i * blk, t1 = (t0 + blk < L) ? t0 + blk : L;
            for (int j = 0; j <= i; ++j) out[(size_t)i * NBmax + j] = 0.0;
            for (int h = 0; h < G; ++h) {
                const uint16_t* qh = q + ((size_t)b * Hq + (size_t)kvh * G + h) * Lmax * D;
                for (int d = 0; d < D; ++d) {
                    double acc = 0.0;
                    for (int t = t0; t < t1; ++t) acc += bf16_to_double(qh[(size_t)t * D + d]);
                    qbar[d] = acc / (double)(t1 - t0);
                }
                for (int e = 0; e < dg; ++e) {
                    double acc = 0.0;
                    for (int d = 0; d < D; ++d) acc += qbar[d] * (double)W[(size_t)e * D + d];
                    qg[e] = acc;
                }
                for (int j = 0; j <= i; ++j) {
                    const double* kp = kpool + (size_t)row * NBmax * dg + (size_t)j * dg;
                    double acc = 0.0;
                    for (int e = 0; e < dg; ++e) acc += qg[e] * kp[e];
                    out[(size_t)i * NBmax + j] += acc * inv_sqrt_dg / (double)G;
                }
            }
        }
        free(qbar);
        free(qg);
    }
}

/* Selection of each query block i < NB_b: block i itself plus the top
 * min(k, i + 1) - 1 of blocks 0 .. i-1 (higher score, then lower index),
 * ascending; k = budget / blk. block_idx [B, Hkv, NBmax, kmax] (-1 padded),
 * num_selected [B, Hkv, NBmax] (0 for i >= NB_b). */
void oracle_prefill_select(const oracle_dims* dm, const double* scores, const int32_t* seq_lens,
                           int32_t budget_tokens, int32_t* block_idx, int32_t* num_selected) {
    const int B = dm->batch, Hkv = dm->num_kv_heads, blk = dm->block_size;
    const int NBmax = num_blocks(dm->max_seq_len, blk);
    const int kmax = budget_tokens / blk;
    for (int row = 0; row < B * Hkv; ++row) {
        const int NB = num_blocks(seq_lens[row / Hkv], blk);
        for (int i = 0; i < NBmax; ++i) {
            int32_t* out = block_idx + ((size_t)row * NBmax + i) * kmax;
            for (int x = 0; x < kmax; ++x) out[x] = -1;
            int32_t* ns = num_selected + (size_t)row * NBmax + i;
            if (i >= NB) { *ns = 0; continue; }
            const double* s = scores + ((size_t)row * NBmax + i) * NBmax;
            const int ki = kmax < i + 1 ? kmax : i + 1;
            scored_block* cand = (scored_block*)malloc(sizeof(scored_block) * (size_t)(i > 0 ? i : 1));
            for (int j = 0; j < i; ++j) { cand[j].score = s[j]; cand[j].index = j; }
            qsort(cand, (size_t)i, sizeof(scored_block), by_score_then_index);
            int n = 0;
            for (int x = 0; x < ki - 1; ++x) out[n++] = cand[x].index;
            qsort(out, (size_t)n, sizeof(int32_t), ascending_int);
            out[n] = i;
            *ns = n + 1;
            free(cand);
        }
    }
}

/* Causal block-sparse attention: query token t < L_b of query block i = t/blk
 * and head h attends to the tokens u <= t (u < L_b) of the kept blocks of
 * (b, kvh, i):  out = softmax(q_t . K_u * scale) V_u,  lse = log sum exp.
 * Rows t >= L_b: out 0, lse -inf. out [B, Hq, Lmax, D], lse [B, Hq, Lmax].
 * Indices outside [0, i] are skipped. sm_scale <= 0 means 1/sqrt(D). */
void oracle_prefill_attend(const oracle_dims* dm, const uint16_t* q, const uint16_t* k_cache,
                           const uint16_t* v_cache, const int32_t* seq_lens, const int32_t* block_idx,
                           const int32_t* num_selected, int32_t kmax, double sm_scale, double* out, double* lse) {
    const int B = dm->batch, Hq = dm->num_q_heads, Hkv = dm->num_kv_heads;
    const int D = dm->head_dim, blk = dm->block_size, Lmax = dm->max_seq_len;
    const int NBmax = num_blocks(Lmax, blk);
    const int G = Hq / Hkv;
    const double scale = (sm_scale > 0.0) ? sm_scale : 1.0 / sqrt((double)D);
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < B * Hq; ++bh) {
        const int b = bh / Hq, hq = bh % Hq, kvh = hq / G;
        const int row = b * Hkv + kvh;
        const int L = seq_lens[b];
        double* z = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
        int32_t* tok = (int32_t*)malloc(sizeof(int32_t) * (size_t)(L > 0 ? L : 1));
        for (int t = 0; t < Lmax; ++t) {
            double* o = out + ((size_t)bh * Lmax + t) * D;
            for (int d = 0; d < D; ++d) o[d] = 0.0;
            if (t >= L) { lse[(size_t)bh * Lmax + t] = -INFINITY; continue; }
            const int i = t / blk;
            const int32_t* idx = block_idx + ((size_t)row * NBmax + i) * kmax;
            const int nsel = num_selected[(size_t)row * NBmax + i];
            int n = 0;
            for (int x = 0; x < nsel; ++x) {
                const int j = idx[x];
                if (j < 0 || j > i) continue;
                for (int u = j * blk; u < (j + 1) * blk && u <= t && u < L; ++u) tok[n++] = u;
            }
            const uint16_t* qt = q + ((size_t)bh * Lmax + t) * D;
            double m = -INFINITY;
            for (int x = 0; x < n; ++x) {
                const uint16_t* ku = k_cache + ((size_t)row * Lmax + tok[x]) * D;
                double acc = 0.0;
                for (int d = 0; d < D; ++d) acc += bf16_to_double(qt[d]) * bf16_to_double(ku[d]);
                z[x] = acc * scale;
                if (z[x] > m) m = z[x];
            }
            if (n == 0) { lse[(size_t)bh * Lmax + t] = -INFINITY; continue; }
            double den = 0.0;
            for (int x = 0; x < n; ++x) {
                const double p = exp(z[x] - m);
                den += p;
                const uint16_t* vu = v_cache + ((size_t)row * Lmax + tok[x]) * D;
                for (int d = 0; d < D; ++d) o[d] += p * bf16_to_double(vu[d]);
            }
            for (int d = 0; d < D; ++d) o[d] /= den;
            lse[(size_t)bh * Lmax + t] = m + log(den);
        }
        free(z);
        free(tok);
    }
}
