// gate_variants.cu -- other readings of the gate: how the G query heads of a
// group are combined into one block score, and threshold selection.
//
// "SeerAttention-R: Sparse Attention Adaptation for Long Reasoning"
// (abstract) scores blocks from the un-pooled decode query with the gate of
// "SeerAttention" (abstract: pooled K through a linear layer, multiplied with
// the projected query) and keeps blocks under a token budget. Neither page
// says how a GQA group's heads share one score, nor whether a threshold can
// replace the budget; these are the alternatives to the mean gate and the
// top-k of gate_scores.cu / select_blocks.cu:
//
//   s_h[j] = (W_q q_h) . kpool[b, kvh, j] / sqrt(dg)        every head on its own
//   mean:          s[j] = (1/G) sum_h s_h[j]
//   max:           s[j] = max_h s_h[j]
//   softmax mean:  s[j] = (1/G) sum_h exp(s_h[j]) / sum_{i < NB_b} exp(s_h[i])
//   threshold:     block NB_b - 1, plus the candidates with s >= tau, at most
//                  k_b - 1 of them (the highest, equal scores to the lower index)
//
// Scores: a cluster of CTAs per (b, kv head) row shares the group's projected
// queries through distributed shared memory and splits the row; lane quads
// score pooled-K rows (the order of gate_core.cuh's quad_row_dot); the
// softmax mean takes three passes over its chunk (max, sum, scores), the
// later ones L2-resident. Threshold selection: one CTA per row.
#include <cuda_bf16.h>

#include <cooperative_groups.h>

#include "gate_core.cuh"
#include "seer_launch.h"

namespace cg = cooperative_groups;

namespace seer {
namespace {

constexpr int kAggThreads = 256;
constexpr int kAggWarps = kAggThreads / 32;
constexpr int kMaxG = 8;
constexpr int kMaxCluster = 8;

// A thread-block cluster of C CTAs per row: each CTA projects dg / C
// components of every head's query and the cluster exchanges them through
// distributed shared memory; each CTA then scores its own contiguous chunk of
// the row. The softmax mean combines each head's chunk maxima, then chunk sums,
// across the cluster the same way.
template <int D, int DG>
__global__ void __launch_bounds__(kAggThreads)
    gate_scores_agg_kernel(const __nv_bfloat16* __restrict__ q, const float* __restrict__ w_q,
                           const float* __restrict__ kpool, const int32_t* __restrict__ seq_lens, int Hq, int Hkv,
                           int Lmax, int blk, int NBmax, int agg, float* __restrict__ scores) {
    __shared__ __align__(16) float qh[kMaxG][D];
    __shared__ float qg_part[kMaxG][DG];          // components this CTA projects
    __shared__ __align__(16) float qg[kMaxG][DG];
    __shared__ float red[kAggWarps][kMaxG];
    __shared__ float part[kMaxG];                 // this CTA's per-head max, then sum (read by the cluster)
    __shared__ float hmax[kMaxG], hsum[kMaxG];
    cg::cluster_group cluster = cg::this_cluster();
    const int csize = (int)cluster.num_blocks();
    const int crank = (int)cluster.block_rank();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = lane >> 2, qlane = lane & 3;
    const int row = blockIdx.y;
    const int b = row / Hkv, kvh = row - b * Hkv;
    const int G = Hq / Hkv;
    const int NB = (clamp_len(seq_lens[b], Lmax) + blk - 1) / blk;
    const float inv_sqrt_dg = 1.0f / sqrtf((float)DG);

    for (int x = tid; x < G * D; x += kAggThreads)
        qh[x / D][x % D] = __bfloat162float(q[((size_t)b * Hq + (size_t)kvh * G) * D + x]);
    __syncthreads();
    const float* W = w_q + (size_t)kvh * DG * D;
    const int per_e = DG / csize;
    for (int e = crank * per_e + warp; e < (crank + 1) * per_e; e += kAggWarps) {
        float wv[D / 32];
#pragma unroll
        for (int u = 0; u < D / 32; ++u) wv[u] = W[(size_t)e * D + lane + 32 * u];
        for (int h = 0; h < G; ++h) {
            float acc = 0.f;
#pragma unroll
            for (int u = 0; u < D / 32; ++u) acc = fmaf(wv[u], qh[h][lane + 32 * u], acc);
            acc = warp_sum(acc);
            if (lane == 0) qg_part[h][e] = acc;
        }
    }
    cluster.sync();
    for (int x = tid; x < G * DG; x += kAggThreads) {
        const int h = x / DG, e = x - h * DG;
        qg[h][e] = *cluster.map_shared_rank(&qg_part[h][e], e / per_e);
    }
    cluster.sync();  // remote reads done before qg_part could be left behind

    const int per = (NB + csize - 1) / csize;
    const int j0 = crank * per, j1 = min(NB, j0 + per);
    const float* kp = kpool + (size_t)row * NBmax * DG;
    float* out = scores + (size_t)row * NBmax;
    auto head_score = [&](int j, int h) { return quad_row_dot<DG>(kp + (size_t)j * DG, j, qg[h], qlane) * inv_sqrt_dg; };
    if (agg == 2) {
        // pass 0: each head's max over the row; pass 1: its sum of exponentials
        for (int pass = 0; pass < 2; ++pass) {
            float acc[kMaxG];
#pragma unroll
            for (int h = 0; h < kMaxG; ++h) acc[h] = pass == 0 ? -INFINITY : 0.f;
            for (int jb = j0 + warp * 8; jb < j1; jb += kAggWarps * 8) {
                const int j = min(jb + quad, j1 - 1);
                const bool live = jb + quad < j1;
#pragma unroll
                for (int h = 0; h < kMaxG; ++h) {
                    if (h >= G) break;
                    const float sc = head_score(j, h);
                    if (live) acc[h] = pass == 0 ? fmaxf(acc[h], sc) : acc[h] + expf(sc - hmax[h]);
                }
            }
#pragma unroll
            for (int h = 0; h < kMaxG; ++h) {
                if (h >= G) break;
                const float v = pass == 0 ? warp_max(acc[h]) : warp_sum(qlane == 0 ? acc[h] : 0.f);
                if (lane == 0) red[warp][h] = v;
            }
            __syncthreads();
            if (tid < G) {
                float v = pass == 0 ? -INFINITY : 0.f;
                for (int w = 0; w < kAggWarps; ++w) v = pass == 0 ? fmaxf(v, red[w][tid]) : v + red[w][tid];
                part[tid] = v;
            }
            cluster.sync();
            if (tid < G) {
                float v = pass == 0 ? -INFINITY : 0.f;
                for (int c = 0; c < csize; ++c) {
                    const float pc = *cluster.map_shared_rank(&part[tid], c);
                    v = pass == 0 ? fmaxf(v, pc) : v + pc;
                }
                if (pass == 0) hmax[tid] = v;
                else hsum[tid] = v;
            }
            cluster.sync();  // remote reads of `part` done before it is rewritten or the CTA exits
        }
    }
    for (int jb = j0 + warp * 8; jb < j1; jb += kAggWarps * 8) {
        const int j = min(jb + quad, j1 - 1);
        float a = agg == 1 ? -INFINITY : 0.f;
#pragma unroll
        for (int h = 0; h < kMaxG; ++h) {
            if (h >= G) break;
            const float sc = head_score(j, h);
            if (agg == 1) a = fmaxf(a, sc);
            else if (agg == 2) a += expf(sc - hmax[h]) / hsum[h];
            else a += sc;
        }
        if (agg != 1) a /= (float)G;
        if (qlane == 0 && jb + quad < j1) out[j] = a;
    }
}

constexpr int kSelThreads = 256;

// Threshold selection: m = min(k_b - 1, #{candidates with score >= tau}); the
// top m of all candidates are then exactly the m highest scoring at least tau,
// so select_row's top-k with k = m + 1 gives the list.
__global__ void __launch_bounds__(kSelThreads)
    select_threshold_kernel(const float* __restrict__ scores, const int32_t* __restrict__ seq_lens, int Hkv, int Lmax,
                            int blk, int NBmax, int kmax, float tau, int32_t* __restrict__ block_idx,
                            int32_t* __restrict__ num_selected) {
    extern __shared__ uint32_t keys[];  // [NBmax]
    __shared__ SelectSmem<kSelThreads> sm;
    const int row = blockIdx.x, tid = threadIdx.x;
    const int L = clamp_len(seq_lens[row / Hkv], Lmax);
    const int NB = (L + blk - 1) / blk;
    const float* s = scores + (size_t)row * NBmax;
    int32_t* out = block_idx + (size_t)row * kmax;
    int mine = 0;
    for (int i = tid; i < NB - 1; i += kSelThreads) {
        keys[i] = order_key(s[i]);
        mine += s[i] >= tau;
    }
    int cnt = 0;
    {
        // block sum of `mine` (counts fit in int)
        __shared__ int part[kSelThreads / 32];
        int v = mine;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if ((tid & 31) == 0) part[tid >> 5] = v;
        __syncthreads();
        for (int w = 0; w < kSelThreads / 32; ++w) cnt += part[w];
    }
    const int kb = kmax < NB ? kmax : NB;
    const int m = NB == 0 ? 0 : min(kb - 1, cnt);
    const int keep = NB == 0 ? 0 : m + 1;
    if (tid == 0) num_selected[row] = keep;
    for (int p = keep + tid; p < kmax; p += kSelThreads) out[p] = -1;
    if (NB > 0) select_row<kSelThreads>(keys, NB, keep, out, sm);
}

template <int D, int DG>
cudaError_t agg_impl(const Shape& s, const void* q, const float* w_q, const float* kpool, const int32_t* seq_lens,
                     int agg, float* scores, int csize, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(csize, s.B * s.Hkv, 1);
    cfg.blockDim = dim3(kAggThreads, 1, 1);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = csize;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, gate_scores_agg_kernel<D, DG>, static_cast<const __nv_bfloat16*>(q),
                                             w_q, kpool, seq_lens, s.Hq, s.Hkv, s.Lmax, s.blk, s.NBmax, agg, scores);
    if (e != cudaSuccess) (void)cudaGetLastError();  // a rejected launch must not leak into the next call
    return e;
}

}  // namespace

cudaError_t launch_gate_scores_agg(const Shape& s, const void* q, const float* w_q, const float* kpool,
                                   const int32_t* seq_lens, int agg, float* scores, int num_sms, cudaStream_t stream) {
    const int rows = s.B * s.Hkv;
    int csize = 1;  // enough CTAs for every SM, at least 32 blocks per CTA
    while (csize < kMaxCluster && rows * csize < 2 * num_sms && s.NBmax / (2 * csize) >= 32) csize *= 2;
    if (s.D == 128 && s.dg == 128) return agg_impl<128, 128>(s, q, w_q, kpool, seq_lens, agg, scores, csize, stream);
    if (s.D == 128 && s.dg == 64) return agg_impl<128, 64>(s, q, w_q, kpool, seq_lens, agg, scores, csize, stream);
    if (s.D == 64 && s.dg == 128) return agg_impl<64, 128>(s, q, w_q, kpool, seq_lens, agg, scores, csize, stream);
    if (s.D == 64 && s.dg == 64) return agg_impl<64, 64>(s, q, w_q, kpool, seq_lens, agg, scores, csize, stream);
    return cudaErrorInvalidValue;
}

cudaError_t launch_select_threshold(const Shape& s, const float* scores, const int32_t* seq_lens, int kmax, float tau,
                                    int32_t* block_idx, int32_t* num_selected, cudaStream_t stream) {
    const size_t smem = (size_t)s.NBmax * sizeof(uint32_t);
    if (smem > 16 * 1024) {  // more than the default limit safely leaves beside the static scratch
        static bool attr_done = false;
        if (!attr_done) {
            cudaError_t e = cudaFuncSetAttribute(select_threshold_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 16384 * 4);
            if (e != cudaSuccess) return e;
            attr_done = true;
        }
    }
    select_threshold_kernel<<<s.B * s.Hkv, kSelThreads, smem, stream>>>(scores, seq_lens, s.Hkv, s.Lmax, s.blk,
                                                                        s.NBmax, kmax, tau, block_idx, num_selected);
    return cudaGetLastError();
}

}  // namespace seer
