// select_blocks.cu -- kept blocks under a token budget.
//
// "SeerAttention-R: Sparse Attention Adaptation for Long Reasoning"
// (abstract) decodes with a fixed token budget (4K) at block sizes 64/128.
// Row (b, kvh) keeps the open last block NB_b - 1 plus the k_b - 1
// highest-scoring blocks among 0 .. NB_b - 2 (k_b = min(budget/blk, NB_b)),
// equal scores going to the lower index, written in ascending order.
//
// One CTA per row. Scores become order-preserving 32-bit keys in shared
// memory; an MSB-first radix select (4 passes of 8 bits, warp-aggregated
// shared-memory histograms) finds the threshold key tau of the (k_b-1)-th
// largest score and how many keys equal to tau are needed. A block-wide scan
// in index order then ranks the tau-ties (lowest indices win) and compacts
// the kept indices, which come out ascending by construction.
#include "seer_device.cuh"
#include "seer_launch.h"

namespace seer {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;

// Monotone map float -> uint32 (a < b  <=>  key(a) < key(b)); -0 is folded
// onto +0 and NaN onto the smallest key.
__device__ __forceinline__ uint32_t order_key(float f) {
    if (f == 0.f) f = 0.f;
    const uint32_t u = __float_as_uint(f);
    if ((u & 0x7fffffffu) > 0x7f800000u) return 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive block-wide prefix sum of one value per thread; also returns the total.
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_tot, int& total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int t = lane < kWarps ? warp_tot[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, t, o);
            if (lane >= o) t += y;
        }
        if (lane < kWarps) warp_tot[lane] = t;  // inclusive warp totals
    }
    __syncthreads();
    total = warp_tot[kWarps - 1];
    const int before = warp == 0 ? 0 : warp_tot[warp - 1];
    __syncthreads();  // warp_tot is reused by the next scan
    return before + x - v;
}

__global__ void __launch_bounds__(kThreads)
    select_blocks_kernel(const float* __restrict__ scores, const int32_t* __restrict__ seq_lens, int Hkv, int Lmax,
                         int blk, int NBmax, int kmax, int32_t* __restrict__ block_idx,
                         int32_t* __restrict__ num_selected) {
    extern __shared__ uint32_t keys[];  // [NBmax]
    __shared__ int hist[256];
    __shared__ int warp_tot[kWarps];
    __shared__ int s_bucket, s_rem;

    const int row = blockIdx.x;
    const int b = row / Hkv;
    const int tid = threadIdx.x;
    const int L = clamp_len(seq_lens[b], Lmax);
    const int NB = (L + blk - 1) / blk;
    const int kb = kmax < NB ? kmax : NB;
    int32_t* out = block_idx + (size_t)row * kmax;
    for (int p = (kb > 0 ? kb : 0) + tid; p < kmax; p += kThreads) out[p] = -1;
    if (tid == 0) num_selected[row] = kb;
    if (NB == 0) return;

    const int ncand = NB - 1;   // blocks 0 .. NB-2 compete; NB-1 is always kept
    const int m = kb - 1;       // how many of them to keep
    if (m >= ncand) {           // everything fits in the budget
        for (int j = tid; j < NB; j += kThreads) out[j] = j;
        return;
    }
    if (m == 0) {
        if (tid == 0) out[0] = NB - 1;
        return;
    }

    const float* s = scores + (size_t)row * NBmax;
    for (int i = tid; i < ncand; i += kThreads) keys[i] = order_key(s[i]);
    __syncthreads();

    // ---- radix select of the m-th largest key
    uint32_t prefix = 0, mask = 0;
    int rem = m;
    const int lane = tid & 31;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = tid; i < 256; i += kThreads) hist[i] = 0;
        __syncthreads();
        for (int base = 0; base < ncand; base += kThreads) {
            const int i = base + tid;
            const bool act = i < ncand && (keys[i] & mask) == prefix;
            const int bucket = act ? (int)((keys[i] >> shift) & 0xffu) : -1;
            const unsigned peers = __match_any_sync(0xffffffffu, bucket);
            if (act && lane == __ffs(peers) - 1) atomicAdd(&hist[bucket], __popc(peers));
        }
        __syncthreads();
        if (tid < 32) {
            // lane l owns buckets 255-8l down to 248-8l (descending)
            int c[8], cnt = 0;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                c[u] = hist[255 - 8 * lane - u];
                cnt += c[u];
            }
            int incl = cnt;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            const int excl = incl - cnt;
            if (excl < rem && rem <= incl) {
                int run = excl;
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    if (run + c[u] >= rem) {
                        s_bucket = 255 - 8 * lane - u;
                        s_rem = rem - run;
                        break;
                    }
                    run += c[u];
                }
            }
        }
        __syncthreads();
        prefix |= (uint32_t)s_bucket << shift;
        mask |= 0xffu << shift;
        rem = s_rem;
        __syncthreads();
    }
    const uint32_t tau = prefix;  // keys > tau are kept; of keys == tau, the first `rem` by index

    // ---- rank the ties and compact, in index order (thread t owns a contiguous range)
    const int per = (ncand + kThreads - 1) / kThreads;
    const int i_lo = tid * per;
    const int i_hi = min(ncand, i_lo + per);
    int n_eq = 0;
    for (int i = i_lo; i < i_hi; ++i) n_eq += keys[i] == tau;
    int total;
    int eq_before = block_exclusive_scan(n_eq, warp_tot, total);
    int n_sel = 0;
    {
        int eq = eq_before;
        for (int i = i_lo; i < i_hi; ++i) {
            const uint32_t k = keys[i];
            n_sel += (k > tau) || (k == tau && eq++ < rem);
        }
    }
    int pos = block_exclusive_scan(n_sel, warp_tot, total);
    {
        int eq = eq_before;
        for (int i = i_lo; i < i_hi; ++i) {
            const uint32_t k = keys[i];
            if ((k > tau) || (k == tau && eq++ < rem)) out[pos++] = i;
        }
    }
    if (tid == 0) out[m] = NB - 1;
}

}  // namespace

cudaError_t launch_select_blocks(const Shape& s, const float* scores, const int32_t* seq_lens, int kmax,
                                 int32_t* block_idx, int32_t* num_selected, cudaStream_t stream) {
    const size_t smem = (size_t)s.NBmax * sizeof(uint32_t);
    if (smem > 48 * 1024) {
        static bool attr_done = false;
        if (!attr_done) {
            cudaError_t e = cudaFuncSetAttribute(select_blocks_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 64 * 1024 + 1024);
            if (e != cudaSuccess) return e;
            attr_done = true;
        }
    }
    select_blocks_kernel<<<s.B * s.Hkv, kThreads, smem, stream>>>(scores, seq_lens, s.Hkv, s.Lmax, s.blk, s.NBmax,
                                                                  kmax, block_idx, num_selected);
    return cudaGetLastError();
}

}  // namespace seer
