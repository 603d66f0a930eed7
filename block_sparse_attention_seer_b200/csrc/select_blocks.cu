// select_blocks.cu -- kept blocks under a token budget.
//
// "SeerAttention-R: Sparse Attention Adaptation for Long Reasoning"
// (abstract) decodes with a fixed token budget (4K) at block sizes 64/128.
// Row (b, kvh) keeps the open last block NB_b - 1 plus the k_b - 1
// highest-scoring blocks among 0 .. NB_b - 2 (k_b = min(budget/blk, NB_b)),
// equal scores going to the lower index, written in ascending order.
//
// One CTA per row (select_row, gate_core.cuh): the scores become
// order-preserving 32-bit keys in shared memory, a value histogram narrows
// down the last kept key, and a scan in index order writes the kept set,
// ascending by construction.
#include "gate_core.cuh"
#include "seer_launch.h"

namespace seer {
namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads)
    select_blocks_kernel(const float* __restrict__ scores, const int32_t* __restrict__ seq_lens, int Hkv, int Lmax,
                         int blk, int NBmax, int kmax, int32_t* __restrict__ block_idx,
                         int32_t* __restrict__ num_selected) {
    after_prior_grid();
    extern __shared__ uint32_t keys[];  // [NBmax]
    __shared__ SelectSmem<kThreads> sm;
    const int row = blockIdx.x;
    const int L = clamp_len(seq_lens[row / Hkv], Lmax);
    const int NB = (L + blk - 1) / blk;
    if (threadIdx.x == 0) num_selected[row] = kmax < NB ? kmax : NB;
    const float* s = scores + (size_t)row * NBmax;
    for (int i = threadIdx.x; i < NB - 1; i += kThreads) keys[i] = order_key(s[i]);
    __syncthreads();
    select_row<kThreads>(keys, NB, kmax, block_idx + (size_t)row * kmax, sm);
}

}  // namespace

cudaError_t launch_select_blocks(const Shape& s, const float* scores, const int32_t* seq_lens, int kmax,
                                 int32_t* block_idx, int32_t* num_selected, cudaStream_t stream) {
    const int rows = s.B * s.Hkv;
    const size_t smem = (size_t)s.NBmax * sizeof(uint32_t);
    if (smem > 16 * 1024) {  // more than the default limit safely leaves beside the static scratch
        static bool attr_done = false;
        if (!attr_done) {
            cudaError_t e = cudaFuncSetAttribute(select_blocks_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 16384 * 4);
            if (e != cudaSuccess) return e;
            attr_done = true;
        }
    }
    return launch_after_prior(select_blocks_kernel, dim3(rows), dim3(kThreads), smem, stream, nullptr, scores,
                              seq_lens, s.Hkv, s.Lmax, s.blk, s.NBmax, kmax, block_idx, num_selected);
}

}  // namespace seer
