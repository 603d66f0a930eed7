// kpool_update.cu -- pooled-and-projected K per KV block, the key side of the
// gate of "SeerAttention: Learning Intrinsic Sparse Attention in Your LLMs"
// (abstract: K is pooled along the sequence dimension and passed through a
// learnable linear layer), kept as a per-block cache so a decode step only
// refreshes the open last block.
//
//   kpool[b,kvh,j,:] = W_k[kvh] . mean_{t in block j, t < L_b} K[b,kvh,t,:]
//
// One CTA (128 threads) per (row, chunk); it walks blocks j = j_first + chunk,
// + chunks, ... below NB_b. The pool reads each block's tokens with 16-byte
// vector loads and accumulates in fp32 in a fixed order; the projection is a
// warp-per-output-row dot product against W_k (read from L2).
#include "seer_device.cuh"
#include "seer_launch.h"

namespace seer {
namespace {

constexpr int kThreads = 128;

template <int D>
__global__ void __launch_bounds__(kThreads)
    kpool_update_kernel(const __nv_bfloat16* __restrict__ k_cache, const float* __restrict__ w_k,
                        const int32_t* __restrict__ seq_lens, const int32_t* __restrict__ upd_start,
                        float* __restrict__ kpool, int Hkv, int Lmax, int blk, int dg, int NBmax, int chunks) {
    constexpr int kLanesPerRow = D / 8;                 // 16-byte pieces per token row
    constexpr int kRowsPerPass = kThreads / kLanesPerRow;
    __shared__ float red[kRowsPerPass][D];
    __shared__ float pooled[D];

    const int row = blockIdx.y;
    const int b = row / Hkv, kvh = row - b * Hkv;
    const int L = clamp_len(seq_lens[b], Lmax);
    const int NB = (L + blk - 1) / blk;
    int start = upd_start ? upd_start[b] : 0;
    start = start < 0 ? 0 : start;
    const int j_first = start / blk;
    const int tid = threadIdx.x;
    const int rsub = tid / kLanesPerRow, cpart = tid % kLanesPerRow;
    const int warp = tid >> 5, lane = tid & 31;
    const __nv_bfloat16* kr = k_cache + (size_t)row * Lmax * D;
    const float* W = w_k + (size_t)kvh * dg * D;

    for (int j = j_first + (int)blockIdx.x; j < NB; j += chunks) {
        const int t0 = j * blk;
        const int n = min(blk, L - t0);
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int t = rsub; t < n; t += kRowsPerPass) {
            const uint4 v = *reinterpret_cast<const uint4*>(kr + (size_t)(t0 + t) * D + cpart * 8);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                acc[2 * u] += __uint_as_float(w[u] << 16);
                acc[2 * u + 1] += __uint_as_float(w[u] & 0xffff0000u);
            }
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) red[rsub][cpart * 8 + u] = acc[u];
        __syncthreads();
        if (tid < D) {
            float s = 0.f;
#pragma unroll
            for (int r = 0; r < kRowsPerPass; ++r) s += red[r][tid];
            pooled[tid] = s / (float)n;
        }
        __syncthreads();
        constexpr int kVec = D / 32;
        float pv[kVec];
#pragma unroll
        for (int u = 0; u < kVec; ++u) pv[u] = pooled[lane * kVec + u];
        for (int e = warp; e < dg; e += kThreads / 32) {
            const float* we = W + (size_t)e * D + lane * kVec;
            float d = 0.f;
            if constexpr (kVec == 4) {
                const float4 wv = *reinterpret_cast<const float4*>(we);
                d = wv.x * pv[0] + wv.y * pv[1] + wv.z * pv[2] + wv.w * pv[3];
            } else {
                const float2 wv = *reinterpret_cast<const float2*>(we);
                d = wv.x * pv[0] + wv.y * pv[1];
            }
            d = warp_sum(d);
            if (lane == 0) kpool[((size_t)row * NBmax + j) * dg + e] = d;
        }
        __syncthreads();  // red / pooled are reused by the next block
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
    if (s.D == 128)
        kpool_update_kernel<128><<<grid, kThreads, 0, stream>>>(k, w_k, seq_lens, upd_start, kpool, s.Hkv, s.Lmax,
                                                               s.blk, s.dg, s.NBmax, chunks);
    else
        kpool_update_kernel<64><<<grid, kThreads, 0, stream>>>(k, w_k, seq_lens, upd_start, kpool, s.Hkv, s.Lmax,
                                                              s.blk, s.dg, s.NBmax, chunks);
    return cudaGetLastError();
}

}  // namespace seer
