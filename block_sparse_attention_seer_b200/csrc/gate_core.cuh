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
//
// The block list of a row is its last block NB-1 plus the m = kb - 1 largest
// keys among candidates 0 .. NB-2, in the order "larger key first, equal keys
// by lower index". That set is fixed by its last member T = (kT, iT):
// candidate i is kept iff key_i > kT, or key_i == kT and i <= iT.

constexpr int kSelectBins = 2048;
constexpr int kSelectHead = 32;  // list entries select_row can also leave in shared memory
constexpr int kSelectBucket = 64;  // boundary bins up to this size are ranked exactly

template <int kThreads>
struct SelectSmem {
    alignas(16) int hist[kSelectBins];
    alignas(16) uint32_t bkey[kSelectBucket];
    alignas(16) int bidx[kSelectBucket];
    uint32_t wlo[kThreads / 32], whi[kThreads / 32];
    int wsum[kThreads / 32];
    int bstar, bcount, above, bfill;
    uint32_t kT;
    int iT;
};

__device__ __forceinline__ int warp_inclusive_scan(int x) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    return x;
}

// Float value of an order key (inverse of order_key; key 0 gives NaN).
__device__ __forceinline__ float key_value(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Histogram bins over a key range [lo, hi], lo < hi: linear in the float value
// when both ends, their difference and the scale are finite, else linear in
// the key. Either way the bin is monotone in the key (k1 <= k2 => bin(k1) <=
// bin(k2)), bin(lo) = 0 and bin(hi) > 0, so the keys of one bin form a key
// interval that holds fewer distinct keys than [lo, hi].
struct SelectBins {
    uint32_t lo;
    float flo, scale;
    int shift;
    bool by_value;
    __device__ __forceinline__ void set(uint32_t lo_, uint32_t hi_) {
        lo = lo_;
        flo = key_value(lo_);
        const float fhi = key_value(hi_);
        const float w = fhi - flo;
        scale = (float)kSelectBins / w;
        by_value = isfinite(flo) && isfinite(fhi) && isfinite(w) && w > 0.f && isfinite(scale);
        const uint32_t d = hi_ - lo_;
        shift = max(0, 32 - __clz((int)d) - 11);  // (d >> shift) < kSelectBins
    }
    __device__ __forceinline__ int operator()(uint32_t k) const {
        if (by_value) return min(kSelectBins - 1, (int)((key_value(k) - flo) * scale));
        return (int)((k - lo) >> shift);
    }
};

// Called once by every thread of select_row when the first histogram has
// fixed the threshold bin: every candidate whose bin (under `bins`, over the
// full key range) is above `bstar` is kept, whatever the rest of the search
// finds. The default does nothing.
struct NoThreshold {
    __device__ __forceinline__ void operator()(const SelectBins&, int) const {}
};

// Block list of one row. keys[0 .. NB-2] (shared memory) hold the order keys
// of the candidate blocks 0 .. NB-2. Writes the kept indices in ascending
// order to out[0 .. kb-1] (kb = min(kmax, NB): block NB-1 always, plus the
// kb-1 largest keys, equal keys going to the lower index) and -1 to out[kb ..
// kmax). When `head` is given (shared memory, kSelectHead entries), the first
// kSelectHead entries of the list are written there too. Threads 0 ..
// kThreads-1 call it and meet at `sync` (by default the whole CTA); shared
// memory is reused only after a barrier that follows the call.
//
// T is found by narrowing a key range [lo, hi] known to hold it: a histogram
// of the range (SelectBins), a CTA scan of the bins from the top to the bin
// where the count reaches the number still to take, then an exact ranking of
// that bin when it holds at most kSelectBucket keys, else a new range = its
// smallest and largest key. Every step removes at least one distinct key; a
// range of one key value keeps its lowest indices. The common case is a
// single histogram and seven barriers.

template <int kThreads, typename OnThreshold = NoThreshold, typename Sync = CtaSync>
__device__ void select_row(const uint32_t* keys, int NB, int kmax, int32_t* __restrict__ out,
                           SelectSmem<kThreads>& sm, int32_t* head = nullptr,
                           OnThreshold on_threshold = OnThreshold(), Sync sync = Sync()) {
    constexpr int kWarps = kThreads / 32;
    constexpr unsigned kFull = 0xffffffffu;
    constexpr int kBinsPer = (kSelectBins + kThreads - 1) / kThreads;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    auto put = [&](int p, int v) {
        out[p] = v;
        if (head && p < kSelectHead) head[p] = v;
    };
    const int kb = kmax < NB ? kmax : NB;
    for (int p = (kb > 0 ? kb : 0) + tid; p < kmax; p += kThreads) put(p, -1);
    if (NB == 0) return;
    const int ncand = NB - 1;
    const int m = kb - 1;
    if (m >= ncand) {
        for (int j = tid; j < NB; j += kThreads) put(j, j);
        return;
    }
    if (m == 0) {
        if (tid == 0) put(0, NB - 1);
        return;
    }
    // Thread t owns the bins kSelectBins-1 - (t*kBinsPer + q), q < kBinsPer (from the top),
    // the strided candidates t, t + kThreads, ... for order-free passes, and the
    // contiguous candidates [c0, c1) for the passes in index order.
    const int per = (ncand + kThreads - 1) / kThreads;
    const int c0 = min(ncand, tid * per), c1 = min(ncand, c0 + per);
    auto bin_of_q = [&](int q) { return kSelectBins - 1 - (tid * kBinsPer + q); };
    auto clear_bins = [&]() {
#pragma unroll
        for (int q = 0; q < kBinsPer; ++q)
            if (bin_of_q(q) >= 0) sm.hist[bin_of_q(q)] = 0;
    };
    // CTA min / max (one barrier; wlo / whi are read again only after later barriers)
    auto block_min_max = [&](uint32_t a, uint32_t b, uint32_t& glo, uint32_t& ghi) {
        a = __reduce_min_sync(kFull, a);
        b = __reduce_max_sync(kFull, b);
        if (lane == 0) {
            sm.wlo[warp] = a;
            sm.whi[warp] = b;
        }
        sync();
        glo = __reduce_min_sync(kFull, lane < kWarps ? sm.wlo[lane] : 0xffffffffu);
        ghi = __reduce_max_sync(kFull, lane < kWarps ? sm.whi[lane] : 0u);
    };
    // exclusive CTA prefix sum in thread order (one barrier); the total to every thread
    auto block_scan = [&](int v, int& total) {
        const int x = warp_inclusive_scan(v);
        if (lane == 31) sm.wsum[warp] = x;
        sync();
        const unsigned w = lane < kWarps ? (unsigned)sm.wsum[lane] : 0u;
        total = (int)__reduce_add_sync(kFull, w);
        return (int)__reduce_add_sync(kFull, lane < warp ? w : 0u) + x - v;
    };

    clear_bins();
    if (tid == 0) sm.bfill = 0;
    uint32_t lo = 0xffffffffu, hi = 0u;
    for (int i = tid; i < ncand; i += kThreads) {
        lo = min(lo, keys[i]);
        hi = max(hi, keys[i]);
    }
    block_min_max(lo, hi, lo, hi);
    int rem = m;  // how many of the keys inside [lo, hi] are kept
    uint32_t kT;
    int iT;
    bool first_pass = true;
    while (true) {
        if (lo == hi) {  // one key value left: its rem lowest indices
            int c = 0;
            for (int i = c0; i < c1; ++i) c += keys[i] == lo;
            int total;
            const int ex = block_scan(c, total);
            if (ex < rem && rem <= ex + c) {
                int seen = ex;
                for (int i = c0; i < c1; ++i)
                    if (keys[i] == lo && ++seen == rem) sm.iT = i;
            }
            sync();
            kT = lo;
            iT = sm.iT;
            break;
        }
        SelectBins bins;
        bins.set(lo, hi);
        for (int i = tid; i < ncand; i += kThreads) {
            const uint32_t k = keys[i];
            if (k >= lo && k <= hi) atomicAdd(&sm.hist[bins(k)], 1);
        }
        sync();
        int mine = 0;
#pragma unroll
        for (int q = 0; q < kBinsPer; ++q)
            if (bin_of_q(q) >= 0) mine += sm.hist[bin_of_q(q)];
        int total;
        const int ex = block_scan(mine, total);
        if (ex < rem && rem <= ex + mine) {
            int run = ex;
            for (int q = 0; q < kBinsPer && bin_of_q(q) >= 0; ++q) {
                const int c = sm.hist[bin_of_q(q)];
                if (run + c >= rem) {
                    sm.bstar = bin_of_q(q);
                    sm.bcount = c;
                    sm.above = run;
                    break;
                }
                run += c;
            }
        }
        sync();
        const int bstar = sm.bstar, bcount = sm.bcount;
        rem -= sm.above;
        if (first_pass) on_threshold(bins, bstar);  // [lo, hi] is still the full key range
        first_pass = false;
        if (bcount <= kSelectBucket) {
            // gather the bin, then rank each entry against the others: T has rank rem - 1
            for (int i = tid; i < ncand; i += kThreads) {
                const uint32_t k = keys[i];
                if (k >= lo && k <= hi && bins(k) == bstar) {
                    const int at = atomicAdd(&sm.bfill, 1);
                    sm.bkey[at] = k;
                    sm.bidx[at] = i;
                }
            }
            sync();
            if (tid < bcount) {
                const uint32_t mk = sm.bkey[tid];
                const int mi = sm.bidx[tid];
                int rank = 0;
                for (int q = 0; q < bcount; ++q) {
                    const uint32_t ok = sm.bkey[q];
                    rank += ok > mk || (ok == mk && sm.bidx[q] < mi);
                }
                if (rank == rem - 1) {
                    sm.kT = mk;
                    sm.iT = mi;
                }
            }
            sync();
            kT = sm.kT;
            iT = sm.iT;
            break;
        }
        // narrow to the bin's own key range; its bins are cleared for the next step
        clear_bins();
        uint32_t nlo = 0xffffffffu, nhi = 0u;
        for (int i = tid; i < ncand; i += kThreads) {
            const uint32_t k = keys[i];
            if (k >= lo && k <= hi && bins(k) == bstar) {
                nlo = min(nlo, k);
                nhi = max(nhi, k);
            }
        }
        block_min_max(nlo, nhi, lo, hi);
    }
    // ---- compaction in index order
    auto kept = [&](int i) {
        const uint32_t k = keys[i];
        return k > kT || (k == kT && i <= iT);
    };
    int n_sel = 0;
    {
        const int len = c1 - c0;  // read from a rotated start, so the lanes of a warp hit different banks
        int off = len > 0 ? lane % len : 0;
        for (int q = 0; q < len; ++q) {
            n_sel += kept(c0 + off);
            if (++off == len) off = 0;
        }
    }
    int total;
    int pos = block_scan(n_sel, total);
    if (n_sel > 0)
        for (int i = c0; i < c1; ++i)
            if (kept(i)) put(pos++, i);
    if (tid == 0) put(m, NB - 1);
}

}  // namespace seer
