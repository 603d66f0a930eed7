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

constexpr int kPoolThreads = 96;  // the pool runs on 96 threads, whatever the CTA size

template <int D>
struct PoolSmem {
    float red[kPoolThreads / (D / 8)][D];
    float pooled[D];
};

struct CtaSync {
    __device__ __forceinline__ void operator()() const { __syncthreads(); }
};

// pooled[d] = (1/n) sum_{t < n} rows[t, d] for a [BLK x D] bf16 block (n >= 1
// valid rows), accumulated in fp32 in a fixed order by the 96 threads
// first_thread .. first_thread + 95. Every thread that `sync` waits for must
// call it (it synchronises twice, by default the whole CTA); the result is
// in sm.pooled.
template <int D, int BLK, typename Sync = CtaSync>
__device__ __forceinline__ void pool_block_mean(const __nv_bfloat16* __restrict__ rows, int n, PoolSmem<D>& sm,
                                                Sync sync = Sync(), int first_thread = 0) {
    constexpr int kLanesPerRow = D / 8;  // 16-byte pieces per token row
    constexpr int kRowsPerPass = kPoolThreads / kLanesPerRow;
    constexpr int kPasses = (BLK + kRowsPerPass - 1) / kRowsPerPass;
    constexpr int kGroup = 6;            // rows loaded before they are summed
    const int pt = (int)threadIdx.x - first_thread;
    if (pt >= 0 && pt < kPoolThreads) {
        const int rsub = pt / kLanesPerRow, cpart = pt % kLanesPerRow;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int p0 = 0; p0 < kPasses; p0 += kGroup) {
            uint4 v[kGroup];
#pragma unroll
            for (int u = 0; u < kGroup; ++u) {
                const int t = rsub + (p0 + u) * kRowsPerPass;
                v[u] = (p0 + u < kPasses && t < n) ? *reinterpret_cast<const uint4*>(rows + (size_t)t * D + cpart * 8)
                                                    : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int u = 0; u < kGroup; ++u) {
                const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    acc[2 * e] += __uint_as_float(w[e] << 16);
                    acc[2 * e + 1] += __uint_as_float(w[e] & 0xffff0000u);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) sm.red[rsub][cpart * 8 + u] = acc[u];
    }
    sync();
    if (pt >= 0 && pt < kPoolThreads) {
        for (int c = pt; c < D; c += kPoolThreads) {
            float s = 0.f;
#pragma unroll
            for (int r = 0; r < kRowsPerPass; ++r) s += sm.red[r][c];
            sm.pooled[c] = s / (float)n;
        }
    }
    sync();
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

// The same mean for one d, with the G <= 8 head loads issued together; the
// additions happen in the same order as group_query_mean's (same bits).
__device__ __forceinline__ float group_query_mean_at(const __nv_bfloat16* __restrict__ qh, int G, int D, int d) {
    float v[8];
#pragma unroll
    for (int h = 0; h < 8; ++h) v[h] = h < G ? __bfloat162float(qh[(size_t)h * D + d]) : 0.f;
    float s = 0.f;
#pragma unroll
    for (int h = 0; h < 8; ++h)
        if (h < G) s += v[h];
    return s / (float)G;
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

// Score dot of pooled-key row j (DG floats at `row`, in global or shared
// memory) with the projected query qg (shared memory, 16-byte aligned),
// computed by the 4 lanes q = 0..3 of a lane quad. Lane q sums the row's
// 16-byte column groups g = (4c + q + 4j) mod DG/4, c = 0, 1, ..., into one
// partial per float4 component; the quad adds its four partials as
// (p0 + p1) + (p2 + p3). The order depends on j alone, so every kernel that
// scores row j gets the same bits; all 4 lanes return the full dot. When a
// warp's 8 quads take 8 consecutive rows, their shared-memory reads fall in
// distinct banks. All 32 lanes of the warp must call it.
template <int DG>
__device__ __forceinline__ float quad_row_dot(const float* row, int j, const float* qg, int q) {
    constexpr int kGroups = DG / 4;
    constexpr int kPer = kGroups / 4;
    const float4* r4 = reinterpret_cast<const float4*>(row);
    const float4* q4 = reinterpret_cast<const float4*>(qg);
    float ax = 0.f, ay = 0.f, az = 0.f, aw = 0.f;
#pragma unroll
    for (int c = 0; c < kPer; ++c) {
        const int g = (4 * c + q + 4 * j) & (kGroups - 1);
        const float4 v = r4[g];
        const float4 w = q4[g];
        ax = fmaf(v.x, w.x, ax);
        ay = fmaf(v.y, w.y, ay);
        az = fmaf(v.z, w.z, az);
        aw = fmaf(v.w, w.w, aw);
    }
    float s = (ax + ay) + (az + aw);
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    s += __shfl_xor_sync(0xffffffffu, s, 2);
    return s;
}

// Monotone map float -> uint32 (a < b  <=>  key(a) < key(b)); -0 is folded
// onto +0 and NaN onto the smallest key.
__device__ __forceinline__ uint32_t order_key(float f) {
    if (f == 0.f) f = 0.f;
    const uint32_t u = __float_as_uint(f);
    if ((u & 0x7fffffffu) > 0x7f800000u) return 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ---------------------------------------------------------------- selection

// ---------------------------------------------------------------- selection

template <int kThreads>
struct SelectSmem {
    int hist[4096];
    int warp_tot[kThreads / 32];
    int bucket, rem, nbound;
    uint32_t bkey[32];  // keys of a boundary bucket of at most 32 elements
    int bidx[32];
    int taken[32];      // which of them are kept
};

// Exclusive CTA-wide prefix sum of one value per thread (ascending thread
// order); *total gets the sum.
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
// order to out[0 .. kb-1] (kb = min(kmax, NB): block NB-1 always, plus the
// kb-1 largest keys, equal keys going to the lower index) and -1 to out[kb ..
// kmax). Every thread of the CTA must call it.
//
// Radix select from the top with digits of 12, 12 and 8 bits: a histogram of
// the current digit over the keys that match the prefix so far, a CTA scan
// from the largest bucket down to the bucket holding the m-th largest key.
// Block scores spread over many 12-bit buckets, so usually after the first
// pass the boundary bucket holds at most 32 keys: one warp then sorts them
// exactly (key descending, index ascending) and the rest is a compaction in
// index order. Keys that stay equal over all 32 bits are resolved by index.
template <int kThreads>
__device__ void select_row(const uint32_t* keys, int NB, int kmax, int32_t* __restrict__ out,
                           SelectSmem<kThreads>& sm) {
    constexpr int kWarps = kThreads / 32;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
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
    uint32_t prefix = 0, mask = 0;
    int rem = m;          // how many keys still to take inside the current prefix
    bool exact = false;   // boundary resolved by the warp sort
    const int shifts[3] = {20, 8, 0};
    const int widths[3] = {12, 12, 8};
    for (int pass = 0; pass < 3 && !exact; ++pass) {
        const int shift = shifts[pass];
        const int nbins = 1 << widths[pass];
        const uint32_t dmask = (uint32_t)nbins - 1u;
        for (int i = tid; i < nbins; i += kThreads) sm.hist[i] = 0;
        __syncthreads();
        for (int i = tid; i < ncand; i += kThreads) {
            const uint32_t k = keys[i];
            if ((k & mask) == prefix) atomicAdd(&sm.hist[(k >> shift) & dmask], 1);
        }
        __syncthreads();
        // thread t owns a run of bins counted from the top: bins nbins-1-t*per ... downwards
        const int per = (nbins + kThreads - 1) / kThreads;
        int mine = 0;
        for (int q = 0; q < per; ++q) {
            const int bin = nbins - 1 - (tid * per + q);
            if (bin >= 0) mine += sm.hist[bin];
        }
        int total;
        const int above = block_exclusive_scan<kThreads>(mine, sm, total);
        if (above < rem && rem <= above + mine) {
            int run = above;
            for (int q = 0; q < per; ++q) {
                const int bin = nbins - 1 - (tid * per + q);
                const int c = sm.hist[bin];
                if (run + c >= rem) {
                    sm.bucket = bin;
                    sm.rem = rem - run;
                    sm.nbound = c;
                    break;
                }
                run += c;
            }
        }
        __syncthreads();
        prefix |= (uint32_t)sm.bucket << shift;
        mask |= dmask << shift;
        rem = sm.rem;
        const int nbound = sm.nbound;
        __syncthreads();
        if (nbound <= 32 && pass < 2) {
            // gather the boundary bucket and sort it exactly inside one warp
            if (tid == 0) sm.nbound = 0;
            __syncthreads();
            for (int i = tid; i < ncand; i += kThreads) {
                const uint32_t k = keys[i];
                if ((k & mask) == prefix) {
                    const int at = atomicAdd(&sm.nbound, 1);
                    sm.bkey[at] = k;
                    sm.bidx[at] = i;
                }
            }
            __syncthreads();
            if (warp == 0) {
                uint32_t k = lane < nbound ? sm.bkey[lane] : 0u;
                int ix = lane < nbound ? sm.bidx[lane] : 0x7fffffff;
                // bitonic sort of 32 (key, index): larger key first, then lower index; padding last
#pragma unroll
                for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
                    for (int stride = size >> 1; stride > 0; stride >>= 1) {
                        const uint32_t ok = __shfl_xor_sync(0xffffffffu, k, stride);
                        const int oi = __shfl_xor_sync(0xffffffffu, ix, stride);
                        const bool mine_first = (k > ok) || (k == ok && ix < oi);
                        const bool up = ((lane & size) == 0) == ((lane & stride) == 0);
                        if (mine_first != up) {
                            k = ok;
                            ix = oi;
                        }
                    }
                }
                sm.taken[lane] = (lane < rem) ? ix : -1;  // the first `rem` of the sorted bucket
            }
            __syncthreads();
            exact = true;
        }
    }
    // ---- compaction in index order (thread t owns a contiguous range of candidates)
    const uint32_t tau = prefix;  // keys above the boundary prefix are kept
    auto above_bound = [&](uint32_t k) { return (k & mask) > tau; };
    auto kept = [&](int i, uint32_t k, int& eq_seen) {
        if (above_bound(k)) return true;
        if ((k & mask) != tau) return false;
        if (exact) {
#pragma unroll 4
            for (int q = 0; q < 32; ++q)
                if (sm.taken[q] == i) return true;
            return false;
        }
        return eq_seen++ < rem;  // all 32 bits equal: the lowest indices win
    };
    const int per = (ncand + kThreads - 1) / kThreads;
    const int i_lo = tid * per;
    const int i_hi = min(ncand, i_lo + per);
    int total;
    int eq_before = 0;
    if (!exact) {
        int n_eq = 0;
        for (int i = i_lo; i < i_hi; ++i) n_eq += (keys[i] & mask) == tau;
        eq_before = block_exclusive_scan<kThreads>(n_eq, sm, total);
    }
    int n_sel = 0;
    {
        int eq = eq_before;
        for (int i = i_lo; i < i_hi; ++i) n_sel += kept(i, keys[i], eq);
    }
    int pos = block_exclusive_scan<kThreads>(n_sel, sm, total);
    {
        int eq = eq_before;
        for (int i = i_lo; i < i_hi; ++i)
            if (kept(i, keys[i], eq)) out[pos++] = i;
    }
    if (tid == 0) out[m] = NB - 1;
    (void)kWarps;
}

}  // namespace seer
