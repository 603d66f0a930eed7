// prefill.cu -- block-sparse attention over a causal prompt.
//
// "SeerAttention: Learning Intrinsic Sparse Attention in Your LLMs"
// (abstract) pools Q and K along the sequence, passes them through learnable
// linear layers, multiplies the results into block-level gating scores, and
// runs a block-sparse FlashAttention over the kept blocks. With the decode
// gate's readings (mean pooling over valid tokens, one bias-free map per KV
// head, mean over the group's heads, 1/sqrt(dg)) this is, for a prompt of L_b
// tokens with query / key blocks of `blk` tokens:
//
//   gate:   s[b,kvh,i,j] = (W_q qbar_i) . kpool[b,kvh,j] / sqrt(dg),  j <= i,
//           qbar_i = the mean of the group's queries over query block i
//   select: block i itself plus the top min(k, i+1) - 1 of blocks 0 .. i-1
//           (the decode rule on a sequence of i + 1 blocks)
//   attend: token t of query block i, head h: causal softmax attention over
//           the tokens u <= t (u < L_b) of the kept blocks of (b, kvh, i)
//
// prefill_gate_kernel / prefill_select_kernel: one CTA per (row, query block).
// The attention step runs on the tcgen05 tensor cores (prefill_attn.cu).
#include <cuda_bf16.h>

#include "gate_core.cuh"
#include "seer_launch.h"

namespace seer {
namespace {

constexpr int kGateThreads = 256;
constexpr int kGateWarps = kGateThreads / 32;

template <int D, int DG>
__global__ void __launch_bounds__(kGateThreads)
    prefill_gate_kernel(const __nv_bfloat16* __restrict__ q, const float* __restrict__ w_q,
                        const float* __restrict__ kpool, const int32_t* __restrict__ seq_lens, int Hq, int Hkv,
                        int Lmax, int blk, int NBmax, float* __restrict__ scores) {
    __shared__ __align__(16) float part[kGateThreads / D][D];
    __shared__ __align__(16) float qbar[D];
    __shared__ __align__(16) float qg[DG];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int i = blockIdx.x, row = blockIdx.y;
    const int b = row / Hkv, kvh = row - b * Hkv;
    const int G = Hq / Hkv;
    const int L = clamp_len(seq_lens[b], Lmax);
    const int NB = (L + blk - 1) / blk;
    if (i >= NB) return;
    const int t0 = i * blk, t1 = min(t0 + blk, L);
    // group- and block-mean of the queries: thread (d, p) sums tokens t0 + p, t0 + p + P, ...
    constexpr int P = kGateThreads / D;
    {
        const int d = tid % D, p = tid / D;
        float acc = 0.f;
        for (int h = 0; h < G; ++h) {
            const __nv_bfloat16* qh = q + (((size_t)b * Hq + (size_t)kvh * G + h) * Lmax) * D + d;
            for (int t = t0 + p; t < t1; t += P) acc += __bfloat162float(qh[(size_t)t * D]);
        }
        part[p][d] = acc;
    }
    __syncthreads();
    if (tid < D) {
        float acc = 0.f;
        for (int p = 0; p < P; ++p) acc += part[p][tid];
        qbar[tid] = acc / (float)(G * (t1 - t0));
    }
    __syncthreads();
    const float* W = w_q + (size_t)kvh * DG * D;
    for (int e = warp; e < DG; e += kGateWarps) {
        float acc = 0.f;
#pragma unroll
        for (int u = 0; u < D / 32; ++u) acc = fmaf(W[(size_t)e * D + lane + 32 * u], qbar[lane + 32 * u], acc);
        acc = warp_sum(acc);
        if (lane == 0) qg[e] = acc;
    }
    __syncthreads();
    const float inv_sqrt_dg = 1.0f / sqrtf((float)DG);
    const float* kp = kpool + (size_t)row * NBmax * DG;
    float* out = scores + ((size_t)row * NBmax + i) * NBmax;
    const int quad = lane >> 2, qlane = lane & 3;
    for (int j0 = warp * 8; j0 <= i; j0 += kGateWarps * 8) {
        const int j = min(j0 + quad, i);
        const float d = quad_row_dot<DG>(kp + (size_t)j * DG, j, qg, qlane);
        if (qlane == 0 && j0 + quad <= i) out[j] = d * inv_sqrt_dg;
    }
}

constexpr int kSelThreads = 256;

__global__ void __launch_bounds__(kSelThreads)
    prefill_select_kernel(const float* __restrict__ scores, const int32_t* __restrict__ seq_lens, int Hkv, int Lmax,
                          int blk, int NBmax, int kmax, int32_t* __restrict__ block_idx,
                          int32_t* __restrict__ num_selected) {
    extern __shared__ uint32_t keys[];  // [NBmax]
    __shared__ SelectSmem<kSelThreads> sm;
    const int i = blockIdx.x, row = blockIdx.y;
    const int L = clamp_len(seq_lens[row / Hkv], Lmax);
    const int NB = (L + blk - 1) / blk;
    const int NBi = i < NB ? i + 1 : 0;  // query block i sees blocks 0 .. i; i is its "last" block
    const size_t ri = (size_t)row * NBmax + i;
    if (threadIdx.x == 0) num_selected[ri] = kmax < NBi ? kmax : NBi;
    const float* s = scores + ri * NBmax;
    for (int j = threadIdx.x; j < NBi - 1; j += kSelThreads) keys[j] = order_key(s[j]);
    __syncthreads();
    select_row<kSelThreads>(keys, NBi, kmax, block_idx + ri * kmax, sm);
}

}  // namespace

cudaError_t launch_prefill_gate(const Shape& s, const void* q, const float* w_q, const float* kpool,
                                const int32_t* seq_lens, float* scores, cudaStream_t stream) {
    const auto* qb = static_cast<const __nv_bfloat16*>(q);
    const dim3 grid(s.NBmax, s.B * s.Hkv);
#define SEER_PG_CASE(DV, DGV)                                                                                      \
    if (s.D == DV && s.dg == DGV) {                                                                                \
        prefill_gate_kernel<DV, DGV><<<grid, kGateThreads, 0, stream>>>(qb, w_q, kpool, seq_lens, s.Hq, s.Hkv,    \
                                                                        s.Lmax, s.blk, s.NBmax, scores);          \
        return cudaGetLastError();                                                                                 \
    }
    SEER_PG_CASE(128, 128)
    SEER_PG_CASE(128, 64)
    SEER_PG_CASE(64, 128)
    SEER_PG_CASE(64, 64)
#undef SEER_PG_CASE
    return cudaErrorInvalidValue;
}

cudaError_t launch_prefill_select(const Shape& s, const float* scores, const int32_t* seq_lens, int kmax,
                                  int32_t* block_idx, int32_t* num_selected, cudaStream_t stream) {
    const size_t smem = (size_t)s.NBmax * sizeof(uint32_t);
    if (smem > 16 * 1024) {
        static bool attr_done = false;
        if (!attr_done) {
            cudaError_t e = cudaFuncSetAttribute(prefill_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 16384 * 4);
            if (e != cudaSuccess) return e;
            attr_done = true;
        }
    }
    prefill_select_kernel<<<dim3(s.NBmax, s.B * s.Hkv), kSelThreads, smem, stream>>>(
        scores, seq_lens, s.Hkv, s.Lmax, s.blk, s.NBmax, kmax, block_idx, num_selected);
    return cudaGetLastError();
}

}  // namespace seer
