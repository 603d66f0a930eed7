// gate_core.cuh -- the gate's arithmetic as CTA-level device functions, shared
// by the separate kernels (kpool_update, gate_scores, select_blocks) and the
// fused decode-step kernel, so both paths compute bit-identical pooled keys,
// scores and block lists.
//
//  * pool_block_mean: mean of the valid token rows of one K block
//    ("SeerAttention: Learning Intrinsic Sparse Attention in Your LLMs",
//    abstract: K pooled along the sequence);
//  * group_query_mean + warp_matvec_rows: the projected, un-pooled decode
//    query W_q q̄ ("SeerAttention-R: Sparse Attention Adaptation for Long
//    Reasoning", abstract: no query pooling in decode);
//  * gate_dot: one block's score, projected query . projected pooled key;
//  * select_row: the last block plus the top (k_b - 1) others, ties to the
//    lower index, ascending ("SeerAttention-R", abstract: token budget).
#pragma once

#include <type_traits>

#include "seer_device.cuh"

namespace seer {

// ---------------------------------------------------------------- pooling

constexpr int kPoolThreads = 128;  // the pool always uses threads 0..127, whatever the CTA size

template <int D>
struct PoolSmem {
    float red[kPoolThreads / (D / 8)][D];
    float pooled[D];
};

// pooled[d] = (1/n) sum_{t < n} rows[t, d] for a [BLK x D] bf16 block (n >= 1
// valid rows), accumulated in fp32 in a fixed order. Every thread of the CTA
// must call it (it synchronises twice); the result is in sm.pooled.
template <int D, int BLK>
__device__ __forceinline__ void pool_block_mean(const __nv_bfloat16* __restrict__ rows, int n, PoolSmem<D>& sm) {
    constexpr int kLanesPerRow = D / 8;  // 16-byte pieces per token row
    constexpr int kRowsPerPass = kPoolThreads / kLanesPerRow;
    constexpr int kPasses = BLK / kRowsPerPass;
    const int tid = threadIdx.x;
    if (tid < kPoolThreads) {
        const int rsub = tid / kLanesPerRow, cpart = tid % kLanesPerRow;
        uint4 v[kPasses];
#pragma unroll
        for (int ps = 0; ps < kPasses; ++ps) {
            const int t = rsub + ps * kRowsPerPass;
            v[ps] = t < n ? *reinterpret_cast<const uint4*>(rows + (size_t)t * D + cpart * 8)
                          : make_uint4(0u, 0u, 0u, 0u);
        }
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ps = 0; ps < kPasses; ++ps) {
            const uint32_t w[4] = {v[ps].x, v[ps].y, v[ps].z, v[ps].w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                acc[2 * u] += __uint_as_float(w[u] << 16);
                acc[2 * u + 1] += __uint_as_float(w[u] & 0xffff0000u);
            }
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) sm.red[rsub][cpart * 8 + u] = acc[u];
    }
    __syncthreads();
    if (tid < D) {
        float s = 0.f;
#pragma unroll
        for (int r = 0; r < kRowsPerPass; ++r) s += sm.red[r][tid];
        sm.pooled[tid] = s / (float)n;
    }
    __syncthreads();
}

// ---------------------------------------------------------------- query side

// qbar[d] = (1/G) sum_h q[h, d] over the G query heads of the group (threads < D).
template <int D>
__device__ __forceinline__ void group_query_mean(const __nv_bfloat16* __restrict__ qh, int G, float* qbar) {
    const int tid = threadIdx.x;
    if (tid < D) {
        float s = 0.f;
        for (int h = 0; h < G; ++h) s += __bfloat162float(qh[(size_t)h * D + tid]);
        qbar[tid] = s / (float)G;
    }
}

// ---------------------------------------------------------------- score

// Warp-wide dot of a dg-float row with the projected query; the lane holds
// qg[lane*DG/32 .. +DG/32). Returns the full dot on every lane.
template <int DG>
__device__ __forceinline__ float gate_dot(const float4& v, const float (&gv)[DG / 32]) {
    static_assert(DG == 128, "float4 form for dg = 128");
    return warp_sum(v.x * gv[0] + v.y * gv[1] + v.z * gv[2] + v.w * gv[3]);
}
template <int DG>
__device__ __forceinline__ float gate_dot(const float2& v, const float (&gv)[DG / 32]) {
    static_assert(DG == 64, "float2 form for dg = 64");
    return warp_sum(v.x * gv[0] + v.y * gv[1]);
}

template <int DG>
using GateVec = typename std::conditional<DG == 128, float4, float2>::type;

// Monotone map float -> uint32 (a < b  <=>  key(a) < key(b)); -0 is folded
// onto +0 and NaN onto the smallest key.
__device__ __forceinline__ uint32_t order_key(float f) {
    if (f == 0.f) f = 0.f;
    const uint32_t u = __float_as_uint(f);
    if ((u & 0x7fffffffu) > 0x7f800000u) return 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ---------------------------------------------------------------- selection

template <int kThreads>
struct SelectSmem {
    int hist[256];
    int warp_tot[kThreads / 32];
    int bucket, rem;
};

// Exclusive CTA-wide prefix sum of one value per thread; *total gets the sum.
template <int kThreads>
__device__ __forceinline__ int block_exclusive_scan(int v, SelectSmem<kThreads>& sm, int& total) {
    constexpr int kWarps = kThreads / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) sm.warp_tot[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int t = lane < kWarps ? sm.warp_tot[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, t, o);
            if (lane >= o) t += y;
        }
        if (lane < kWarps) sm.warp_tot[lane] = t;  // inclusive warp totals
    }
    __syncthreads();
    total = sm.warp_tot[kWarps - 1];
    const int before = warp == 0 ? 0 : sm.warp_tot[warp - 1];
    __syncthreads();  // warp_tot is reused by the next scan
    return before + x - v;
}

// Block list of one row. keys[0 .. NB-2] (shared memory) hold the order keys
// of the candidate blocks 0 .. NB-2. Writes the kept indices in ascending
// order to out[0 .. kb-1] (kb = min(kmax, NB), block NB-1 always kept, the
// others the kb-1 largest keys, equal keys to the lower index) and -1 to
// out[kb .. kmax). Every thread of the CTA must call it; keys may be left
// unread when the choice is trivial.
template <int kThreads>
__device__ void select_row(const uint32_t* keys, int NB, int kmax, int32_t* __restrict__ out,
                           SelectSmem<kThreads>& sm) {
    const int tid = threadIdx.x, lane = tid & 31;
    const int kb = kmax < NB ? kmax : NB;
    for (int p = (kb > 0 ? kb : 0) + tid; p < kmax; p += kThreads) out[p] = -1;
    if (NB == 0) return;
    const int ncand = NB - 1;  // blocks 0 .. NB-2 compete; NB-1 is always kept
    const int m = kb - 1;      // how many of them to keep
    if (m >= ncand) {          // everything fits in the budget
        for (int j = tid; j < NB; j += kThreads) out[j] = j;
        return;
    }
    if (m == 0) {
        if (tid == 0) out[0] = NB - 1;
        return;
    }
    // ---- MSB-first radix select of the m-th largest key (4 passes of 8 bits)
    uint32_t prefix = 0, mask = 0;
    int rem = m;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = tid; i < 256; i += kThreads) sm.hist[i] = 0;
        __syncthreads();
        for (int base = 0; base < ncand; base += kThreads) {
            const int i = base + tid;
            const bool act = i < ncand && (keys[i] & mask) == prefix;
            const int bucket = act ? (int)((keys[i] >> shift) & 0xffu) : -1;
            const unsigned peers = __match_any_sync(0xffffffffu, bucket);
            if (act && lane == __ffs(peers) - 1) atomicAdd(&sm.hist[bucket], __popc(peers));
        }
        __syncthreads();
        if (tid < 32) {
            // lane l owns buckets 255-8l down to 248-8l (descending)
            int c[8], cnt = 0;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                c[u] = sm.hist[255 - 8 * lane - u];
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
                        sm.bucket = 255 - 8 * lane - u;
                        sm.rem = rem - run;
                        break;
                    }
                    run += c[u];
                }
            }
        }
        __syncthreads();
        prefix |= (uint32_t)sm.bucket << shift;
        mask |= 0xffu << shift;
        rem = sm.rem;
        __syncthreads();
    }
    const uint32_t tau = prefix;  // keys > tau are kept; of keys == tau, the first `rem` by index

    // ---- rank the ties and compact in index order (thread t owns a contiguous range)
    const int per = (ncand + kThreads - 1) / kThreads;
    const int i_lo = tid * per;
    const int i_hi = min(ncand, i_lo + per);
    int n_eq = 0;
    for (int i = i_lo; i < i_hi; ++i) n_eq += keys[i] == tau;
    int total;
    const int eq_before = block_exclusive_scan<kThreads>(n_eq, sm, total);
    int n_sel = 0;
    {
        int eq = eq_before;
        for (int i = i_lo; i < i_hi; ++i) {
            const uint32_t k = keys[i];
            n_sel += (k > tau) || (k == tau && eq++ < rem);
        }
    }
    int pos = block_exclusive_scan<kThreads>(n_sel, sm, total);
    {
        int eq = eq_before;
        for (int i = i_lo; i < i_hi; ++i) {
            const uint32_t k = keys[i];
            if ((k > tau) || (k == tau && eq++ < rem)) out[pos++] = i;
        }
    }
    if (tid == 0) out[m] = NB - 1;
}

}  // namespace seer
