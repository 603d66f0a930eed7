// kpool_update.cu -- pooled-and-projected K per KV block, the key side of the
// gate of "SeerAttention: Learning Intrinsic Sparse Attention in Your LLMs"
// (abstract: K is pooled along the sequence dimension and passed through a
// learnable linear layer), kept as a per-block cache so a decode step only
// refreshes the open last block.
//
//   kpool[b,kvh,j,:] = W_k[kvh] . mean_{t in block j, t < L_b} K[b,kvh,t,:]
//
// One CTA (128 threads) per (row, chunk); it walks blocks j = j_first + chunk,
// + chunks, ... below NB_b. The pool (gate_core.cuh) loads all of a thread's
// token rows with 16-byte vector loads before summing them in fp32 in a fixed
// order; the projection is one warp per output row against W_k, eight rows
// in flight per warp.
#include "gate_core.cuh"
#include "seer_launch.h"

namespace seer {
namespace {

constexpr int kThreads = 128;

template <int D, int BLK>
__global__ void __launch_bounds__(kThreads)
    kpool_update_kernel(const __nv_bfloat16* __restrict__ k_cache, const float* __restrict__ w_k,
                        const int32_t* __restrict__ seq_lens, const int32_t* __restrict__ upd_start,
                        float* __restrict__ kpool, int Hkv, int Lmax, int dg, int NBmax, int chunks) {
    after_prior_grid();
    __shared__ PoolSmem<D> sm;
    const int row = blockIdx.y;
    const int b = row / Hkv, kvh = row - b * Hkv;
    const int L = clamp_len(seq_lens[b], Lmax);
    const int NB = (L + BLK - 1) / BLK;
    int start = upd_start ? upd_start[b] : 0;
    start = start < 0 ? 0 : start;
    const int j_first = start / BLK;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const __nv_bfloat16* kr = k_cache + (size_t)row * Lmax * D;
    const float* W = w_k + (size_t)kvh * dg * D;

    for (int j = j_first + (int)blockIdx.x; j < NB; j += chunks) {
        pool_block_mean<D, BLK>(kr + (size_t)j * BLK * D, min(BLK, L - j * BLK), sm);
        float pv[D / 32];
#pragma unroll
        for (int u = 0; u < D / 32; ++u) pv[u] = sm.pooled[lane * (D / 32) + u];
        float* dst = kpool + ((size_t)row * NBmax + j) * dg;
        warp_matvec_rows<D>(W, pv, warp, dg, kThreads / 32, [&](int e, float x) { dst[e] = x; });
        __syncthreads();  // sm is reused by the next block
    }
}

}  // namespace

cudaError_t launch_kpool_update(const Shape& s, const void* k_cache, const float* w_k, const int32_t* seq_lens,
                                const int32_t* upd_start, float* kpool, int num_sms, cudaStream_t stream) {
    const int rows = s.B * s.Hkv;
    int chunks = (2 * num_sms + rows - 1) / rows;
    if (chunks > s.NBmax) chunks = s.NBmax;
    if (chunks < 1) chunks = 1;
    if (upd_start) chunks = 1 + (chunks > 1);  // a decode refresh touches one block, rarely two
    const dim3 grid(chunks, rows);
    const auto* k = static_cast<const __nv_bfloat16*>(k_cache);
#define SEER_KPOOL(D_, B_)                                                                                       \
    launch_after_prior(kpool_update_kernel<D_, B_>, grid, dim3(kThreads), 0, stream, nullptr, k, w_k, seq_lens,   \
                       upd_start, kpool, s.Hkv, s.Lmax, s.dg, s.NBmax, chunks)
    cudaError_t e;
    if (s.D == 128 && s.blk == 64) e = SEER_KPOOL(128, 64);
    else if (s.D == 128) e = SEER_KPOOL(128, 128);
    else if (s.blk == 64) e = SEER_KPOOL(64, 64);
    else e = SEER_KPOOL(64, 128);
#undef SEER_KPOOL
    return e;
}

}  // namespace seer
