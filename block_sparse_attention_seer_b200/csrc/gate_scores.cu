// gate_scores.cu -- block gating scores from the un-pooled decode query.
//
// "SeerAttention-R: Sparse Attention Adaptation for Long Reasoning"
// (abstract) keeps SeerAttention's gate but removes query pooling, so the
// single decode query is projected as is; "SeerAttention: Learning Intrinsic
// Sparse Attention in Your LLMs" (abstract) multiplies the projected query
// with the projected pooled keys to score each block. Per (b, kvh):
//
//   s[j] = (1/G) sum_h (W_q q_h) . kpool[j] / sqrt(dg)
//        = (W_q qbar) . kpool[j] / sqrt(dg),   qbar = (1/G) sum_h q_h
//
// (the two forms agree by linearity; the second needs one projection). The
// scan over kpool is the HBM cost. A thread-block cluster of C CTAs serves one
// row: each CTA projects dg/C components of W_q qbar, the cluster exchanges
// them through distributed shared memory, and each CTA then scores its own
// contiguous chunk of the row's blocks, one lane quad per block row
// (quad_row_dot, the same summation order as the fused step).
#include <cooperative_groups.h>

#include "gate_core.cuh"
#include "seer_launch.h"

namespace cg = cooperative_groups;

namespace seer {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

template <int D, int DG>
__global__ void __launch_bounds__(kThreads)
    gate_scores_kernel(const __nv_bfloat16* __restrict__ q, const float* __restrict__ w_q,
                       const float* __restrict__ kpool, const int32_t* __restrict__ seq_lens,
                       float* __restrict__ scores, int Hq, int Hkv, int G, int blk, int Lmax, int NBmax) {
    after_prior_grid();
    __shared__ float qbar[D];
    __shared__ float qg_part[DG];  // components this CTA projects (others stay unused)
    __shared__ __align__(16) float qg[DG];

    cg::cluster_group cluster = cg::this_cluster();
    const int csize = (int)cluster.num_blocks();
    const int crank = (int)cluster.block_rank();
    const int row = blockIdx.y;
    const int b = row / Hkv, kvh = row - b * Hkv;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    group_query_mean<D>(q + ((size_t)b * Hq + (size_t)kvh * G) * D, G, qbar);
    __syncthreads();
    constexpr int kVecD = D / 32;
    {
        float qv[kVecD];
#pragma unroll
        for (int u = 0; u < kVecD; ++u) qv[u] = qbar[lane * kVecD + u];
        const int per = DG / csize;
        warp_matvec_rows<D>(w_q + (size_t)kvh * DG * D, qv, crank * per + warp, (crank + 1) * per, kWarps,
                            [&](int e, float x) { qg_part[e] = x; });
    }
    cluster.sync();
    if (tid < DG) {
        const int owner = tid / (DG / csize);
        qg[tid] = *cluster.map_shared_rank(&qg_part[tid], owner);
    }
    cluster.sync();  // remote reads done before any CTA of the cluster moves on or exits

    const int L = clamp_len(seq_lens[b], Lmax);
    const int NB = (L + blk - 1) / blk;
    const int per = (NB + csize - 1) / csize;
    const int j0 = crank * per;
    const int j1 = min(NB, j0 + per);
    // one lane quad per block row, 8 consecutive rows per warp step
    const float inv_sqrt_dg = 1.0f / sqrtf((float)DG);
    const float* kp = kpool + (size_t)row * NBmax * DG;
    float* out = scores + (size_t)row * NBmax;
    const int quad = lane >> 2, qlane = lane & 3;
    for (int jb = j0 + warp * 8; jb < j1; jb += kWarps * 8) {
        const int j = min(jb + quad, j1 - 1);  // lanes past j1 repeat the last row and store nothing
        const float d = quad_row_dot<DG>(kp + (size_t)j * DG, j, qg, qlane);
        if (qlane == 0 && jb + quad < j1) out[j] = d * inv_sqrt_dg;
    }
}

template <int D, int DG>
cudaError_t launch_impl(const Shape& s, const void* q, const float* w_q, const float* kpool,
                        const int32_t* seq_lens, float* scores, int csize, cudaStream_t stream) {
    cudaLaunchAttribute cluster;
    cluster.id = cudaLaunchAttributeClusterDimension;
    cluster.val.clusterDim.x = csize;
    cluster.val.clusterDim.y = 1;
    cluster.val.clusterDim.z = 1;
    return launch_after_prior(gate_scores_kernel<D, DG>, dim3(csize, s.B * s.Hkv, 1), dim3(kThreads, 1, 1), 0, stream,
                              &cluster, static_cast<const __nv_bfloat16*>(q), w_q, kpool, seq_lens, scores, s.Hq,
                              s.Hkv, s.G, s.blk, s.Lmax, s.NBmax);
}

}  // namespace

cudaError_t launch_gate_scores(const Shape& s, const void* q, const float* w_q, const float* kpool,
                               const int32_t* seq_lens, float* scores, int num_sms, cudaStream_t stream) {
    const int rows = s.B * s.Hkv;
    int csize = 1;
    while (csize < 8 && rows * csize < 2 * num_sms && s.NBmax / (2 * csize) >= 32) csize *= 2;
    cudaError_t e;
    if (s.D == 128 && s.dg == 128) e = launch_impl<128, 128>(s, q, w_q, kpool, seq_lens, scores, csize, stream);
    else if (s.D == 128 && s.dg == 64) e = launch_impl<128, 64>(s, q, w_q, kpool, seq_lens, scores, csize, stream);
    else if (s.D == 64 && s.dg == 128) e = launch_impl<64, 128>(s, q, w_q, kpool, seq_lens, scores, csize, stream);
    else e = launch_impl<64, 64>(s, q, w_q, kpool, seq_lens, scores, csize, stream);
    if (e != cudaSuccess) {
        (void)cudaGetLastError();  // a rejected launch must not leak into the next call
        return e;
    }
    return cudaGetLastError();
}

}  // namespace seer
