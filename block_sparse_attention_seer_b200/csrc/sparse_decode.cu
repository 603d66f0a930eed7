// sparse_decode.cu -- block-sparse split-KV flash-decode for sm_100a.
//
// Computes, for every (batch b, KV head kvh) row and each of its G query
// heads, softmax attention over the valid tokens of the kept KV blocks only:
// the "sparse decoding kernel" of "SeerAttention-R: Sparse Attention
// Adaptation for Long Reasoning" (abstract), whose time is meant to scale
// with the kept blocks instead of the context. The pages give no kernel
// design for this GPU; this one is built for B200:
//
//  * persistent grid, one CTA per SM. The kept blocks of all rows, laid end
//    to end (kmax positions per row), are cut into P equal contiguous
//    ranges, one per CTA, so each SM streams the same number of blocks and
//    its copy pipeline never drains between rows. Each (CTA, row) overlap
//    produces one partial (o, lse) "slot"; seer_combine merges slots.
//  * one producer warp: a single lane issues 2-D TMA tile loads (128-byte
//    swizzle) of the whole K and V tile of each kept block straight into a
//    ring of shared-memory stages, with an mbarrier pair per stage; the
//    decode query of a row rides along as a bulk copy with the row's first
//    block. Loads carry an L2 evict-first hint (each tile is read once).
//  * eight consumer warps, each owning a fixed slice of blk/8 tokens of every
//    block. Q K^T and P V run on the tensor cores (mma.sync bf16 -> fp32):
//    the G <= 8 query heads of the group form the M side (padded to 16),
//    tokens and head_dim the N / K sides, operands fetched with ldmatrix
//    (swizzle-matched, conflict-free). Each warp keeps its own online
//    softmax state; the eight states are merged through shared memory at the
//    end of each row segment.
//  * tokens t >= L_b of the partial last block are masked to -inf and their
//    V rows zeroed in shared memory before P V (the cache past L_b may hold
//    anything, NaN included).
//  * every wait is an mbarrier wait with a time limit; on expiry the CTA
//    records an error, writes NaN into the slot it was producing and exits
//    after its own copies have landed.
#include <cfloat>
#include <cmath>

#include "seer_device.cuh"
#include "seer_launch.h"

namespace seer {

// Count of decode CTAs that gave up on a wait (0 in normal operation).
__device__ unsigned int g_decode_wait_failures = 0;

namespace {

constexpr int kConsumerWarps = 8;
constexpr int kConsumerThreads = kConsumerWarps * 32;
constexpr int kThreads = kConsumerThreads + 32;
constexpr int kMaxStages = 8;
constexpr int kSmemLimit = 232448;  // 227 KB of opt-in dynamic shared memory per CTA
constexpr float kLn2 = 0.69314718055994530942f;
constexpr float kLog2e = 1.44269504088896340736f;

template <int D, int BLK>
struct Cfg {
    static constexpr int kTokPerWarp = BLK / kConsumerWarps;  // 8 or 16 tokens of each block
    static constexpr int kNT8 = kTokPerWarp / 8;               // n8 tiles of S per warp
    static constexpr int kBoxes = D / 64;                      // 64-column (128-byte) TMA boxes per tile
    static constexpr int kBoxBytes = BLK * 128;
    static constexpr int kTileBytes = BLK * D * 2;
    static constexpr int kKSteps = D / 16;
    static constexpr int kDTiles = D / 8;
};

struct Params {
    const __nv_bfloat16* q;
    const int32_t* seq_lens;
    const int32_t* block_idx;
    const int32_t* num_selected;
    float* o_part;
    float* lse_part;
    long long V;  // rows * kmax virtual positions
    int Hq, Hkv, G, Lmax, kmax, S, P, nst;
    int stage_bytes, merge_off, info_off, bar_off;
    float scale_log2;  // sm_scale * log2(e)
};

// One row's share of this CTA's range.
struct Segment {
    int row, b, kvh, L, a0, a1, slot, nslots;
    bool last;  // this CTA holds the end of the row's reserved positions
};

__device__ __forceinline__ Segment make_segment(const Params& p, int r, long long g0, long long g1) {
    Segment s;
    const long long rs = (long long)r * p.kmax;
    const int i0 = (int)(g0 > rs ? g0 - rs : 0);
    const int i1 = (int)((g1 - rs) < p.kmax ? (g1 - rs) : p.kmax);
    s.row = r;
    s.b = r / p.Hkv;
    s.kvh = r - s.b * p.Hkv;
    s.L = clamp_len(p.seq_lens[s.b], p.Lmax);
    int n = s.L == 0 ? 0 : p.num_selected[r];
    n = n < 0 ? 0 : (n > p.kmax ? p.kmax : n);
    s.a0 = i0 < n ? i0 : n;
    s.a1 = i1 < n ? i1 : n;
    // CTA that holds virtual position x: the largest c with floor(c*V/P) <= x.
    const int c_first = (int)(((rs + 1) * p.P - 1) / p.V);
    const int c_last = (int)(((rs + p.kmax) * p.P - 1) / p.V);
    s.slot = (int)blockIdx.x - c_first;
    s.nslots = c_last - c_first + 1;
    s.last = (i1 == p.kmax);
    return s;
}

// Byte address of element (token, d0 .. d0+7) of a [BLK x D] bf16 tile stored
// as D/64 TMA boxes of BLK rows x 128 bytes with the 128-byte swizzle (16-byte
// chunk index XOR row mod 8).
template <int BLK>
__device__ __forceinline__ uint32_t swz(uint32_t tile, int tok, int d0) {
    return tile + (uint32_t)((d0 >> 6) * (BLK * 128) + tok * 128 + ((((d0 & 63) >> 3) ^ (tok & 7)) << 4));
}

__device__ __forceinline__ void record_failure(int* abort_flag) {
    if (atomicExch(abort_flag, 1) == 0) atomicAdd(&g_decode_wait_failures, 1u);
}

template <int D, int BLK>
__global__ void __launch_bounds__(kThreads, 1)
    sparse_decode_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                         const Params p) {
    using C = Cfg<D, BLK>;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    unsigned char* base = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                           ~uintptr_t(1023));
    const uint32_t sbase = smem_addr(base);
    float* merge = reinterpret_cast<float*>(base + p.merge_off);
    int* info = reinterpret_cast<int*>(base + p.info_off);
    int* abort_flag = info + kMaxStages;
    const uint32_t bars = sbase + p.bar_off;  // full[0..nst), empty[0..nst), consumer barrier
    auto bar_full = [&](int st) { return bars + 8u * st; };
    auto bar_empty = [&](int st) { return bars + 8u * (p.nst + st); };
    const uint32_t bar_cons = bars + 16u * p.nst;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int st = 0; st < p.nst; ++st) {
            mbar_init(bar_full(st), 1);
            mbar_init(bar_empty(st), kConsumerWarps);
        }
        mbar_init(bar_cons, kConsumerThreads);
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    const long long g0 = (long long)blockIdx.x * p.V / p.P;
    const long long g1 = (long long)(blockIdx.x + 1) * p.V / p.P;
    const int r_begin = (int)(g0 / p.kmax);

    if (warp == kConsumerWarps) {
        // ------------------------------------------------------------ producer warp
        if (lane == 0) {
            prefetch_tensor_map(&tmK);
            prefetch_tensor_map(&tmV);
        }
        const uint64_t policy = l2_policy_evict_first();
        int st = 0;
        uint32_t ph = 0;
        long long issued = 0;
        bool ok = true;
        for (int r = r_begin; ok && (long long)r * p.kmax < g1; ++r) {
            const Segment s = make_segment(p, r, g0, g1);
            if (s.a1 <= s.a0) continue;
            const int NB = (s.L + BLK - 1) / BLK;
            const __nv_bfloat16* qsrc = p.q + ((size_t)s.b * p.Hq + (size_t)s.kvh * p.G) * D;
            const int32_t* list = p.block_idx + (size_t)r * p.kmax;
            for (int i = s.a0; ok && i < s.a1; i += 32) {
                const int jl = (i + lane < s.a1) ? list[i + lane] : -1;
                const int cnt = min(32, s.a1 - i);
                for (int k = 0; ok && k < cnt; ++k) {
                    const int j = __shfl_sync(0xffffffffu, jl, k);
                    const int valid = (j >= 0 && j < NB) ? min(BLK, s.L - j * BLK) : 0;
                    int good = 1;
                    if (lane == 0) {
                        if (!mbar_wait(bar_empty(st), ph ^ 1u)) {
                            good = 0;
                            record_failure(abort_flag);
                        } else {
                            info[st] = valid;
                            const bool first = (i + k == s.a0);
                            const uint32_t fb = bar_full(st);
                            const uint32_t bytes =
                                (valid > 0 ? 2u * C::kTileBytes : 0u) + (first ? (uint32_t)(p.G * D * 2) : 0u);
                            if (bytes) mbar_arrive_expect_tx(fb, bytes);
                            else mbar_arrive(fb);
                            const uint32_t stK = sbase + (uint32_t)st * p.stage_bytes;
                            if (valid > 0) {
                                const int y = r * p.Lmax + j * BLK;
#pragma unroll
                                for (int bx = 0; bx < C::kBoxes; ++bx) {
                                    tma_load_2d(stK + bx * C::kBoxBytes, &tmK, fb, bx * 64, y, policy);
                                    tma_load_2d(stK + C::kTileBytes + bx * C::kBoxBytes, &tmV, fb, bx * 64, y,
                                                policy);
                                }
                            }
                            if (first) bulk_load(stK + 2 * C::kTileBytes, qsrc, (uint32_t)(p.G * D * 2), fb);
                            ++issued;
                        }
                    }
                    ok = __shfl_sync(0xffffffffu, good, 0) != 0;
                    if (ok && ++st == p.nst) {
                        st = 0;
                        ph ^= 1u;
                    }
                }
            }
        }
        if (lane == 0) {
            // Tail: the producer warp leaves only once every copy it issued has
            // landed -- normally by seeing the consumers release the last stages,
            // after a failed wait by seeing the copies complete.
            for (long long it = (issued > p.nst ? issued - p.nst : 0); it < issued; ++it) {
                const int s_it = (int)(it % p.nst);
                const uint32_t par = (uint32_t)((it / p.nst) & 1);
                if (!ok || !mbar_wait(bar_empty(s_it), par)) (void)mbar_wait(bar_full(s_it), par);
            }
        }
        return;
    }

    // ---------------------------------------------------------------- consumer warps
    const int ctid = threadIdx.x;                  // 0 .. 255
    const int g = lane >> 2, tig = lane & 3;       // mma fragment coordinates
    const int tbase = warp * C::kTokPerWarp;       // this warp's token slice of each block
    float* mO = merge;                             // [8][G][D]
    float* mM = merge + kConsumerWarps * p.G * D;  // [8][G]
    float* mL = mM + kConsumerWarps * p.G;         // [8][G]
    int st = 0;
    uint32_t ph = 0, cph = 0;
    bool ok = true;

    for (int r = r_begin; ok && (long long)r * p.kmax < g1; ++r) {
        const Segment s = make_segment(p, r, g0, g1);
        const size_t head0 = (size_t)s.b * p.Hq + (size_t)s.kvh * p.G;
        if (s.a1 > s.a0) {
            float m_run = -INFINITY, l_run = 0.f;
            float o[C::kDTiles][4];
#pragma unroll
            for (int dt = 0; dt < C::kDTiles; ++dt) o[dt][0] = o[dt][1] = o[dt][2] = o[dt][3] = 0.f;
            uint32_t qa[C::kKSteps][2];

            for (int i = s.a0; i < s.a1; ++i) {
                if (!mbar_wait(bar_full(st), ph)) {
                    record_failure(abort_flag);
                    ok = false;
                    break;
                }
                const int valid = info[st];
                const uint32_t stK = sbase + (uint32_t)st * p.stage_bytes;
                const uint32_t stV = stK + C::kTileBytes;
                if (i == s.a0) {
                    const __nv_bfloat16* qs =
                        reinterpret_cast<const __nv_bfloat16*>(base + (size_t)st * p.stage_bytes + 2 * C::kTileBytes);
#pragma unroll
                    for (int kk = 0; kk < C::kKSteps; ++kk) {
                        qa[kk][0] = g < p.G ? *reinterpret_cast<const uint32_t*>(qs + g * D + kk * 16 + 2 * tig) : 0u;
                        qa[kk][1] = g < p.G ? *reinterpret_cast<const uint32_t*>(qs + g * D + kk * 16 + 8 + 2 * tig) : 0u;
                    }
                }
                bool wrote = false;
                if (valid > tbase) {
                    // ---- S = Q K^T over this warp's tokens (rows: heads, cols: tokens)
                    float sacc[C::kNT8][4];
#pragma unroll
                    for (int nt = 0; nt < C::kNT8; ++nt) sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
                    if constexpr (C::kNT8 == 1) {
                        float s2[4] = {0.f, 0.f, 0.f, 0.f};
                        const int mi = lane >> 3;
                        const int tok = tbase + (lane & 7);
#pragma unroll
                        for (int kk2 = 0; kk2 < C::kKSteps / 2; ++kk2) {
                            uint32_t r0, r1, r2, r3;
                            ldmatrix_x4(swz<BLK>(stK, tok, (2 * kk2 + (mi >> 1)) * 16 + (mi & 1) * 8), r0, r1, r2, r3);
                            mma_bf16_16816(sacc[0], qa[2 * kk2][0], 0u, qa[2 * kk2][1], 0u, r0, r1);
                            mma_bf16_16816(s2, qa[2 * kk2 + 1][0], 0u, qa[2 * kk2 + 1][1], 0u, r2, r3);
                        }
#pragma unroll
                        for (int e = 0; e < 4; ++e) sacc[0][e] += s2[e];
                    } else {
                        const int mi = lane >> 3;
                        const int tok = tbase + (mi >> 1) * 8 + (lane & 7);
#pragma unroll
                        for (int kk = 0; kk < C::kKSteps; ++kk) {
                            uint32_t r0, r1, r2, r3;
                            ldmatrix_x4(swz<BLK>(stK, tok, kk * 16 + (mi & 1) * 8), r0, r1, r2, r3);
                            mma_bf16_16816(sacc[0], qa[kk][0], 0u, qa[kk][1], 0u, r0, r1);
                            mma_bf16_16816(sacc[1], qa[kk][0], 0u, qa[kk][1], 0u, r2, r3);
                        }
                    }
                    // ---- online softmax for row g (query head g of the group)
                    float x[C::kNT8][2];
                    float mloc = -INFINITY;
#pragma unroll
                    for (int nt = 0; nt < C::kNT8; ++nt) {
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int t = tbase + nt * 8 + 2 * tig + e;
                            x[nt][e] = (t < valid) ? sacc[nt][e] * p.scale_log2 : -INFINITY;
                            mloc = fmaxf(mloc, x[nt][e]);
                        }
                    }
                    mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, 1));
                    mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, 2));
                    const float m_new = fmaxf(m_run, mloc);
                    const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
                    const float alpha = exp2f(m_run - m_use);
                    float pv[C::kNT8][2];
                    float psum = 0.f;
#pragma unroll
                    for (int nt = 0; nt < C::kNT8; ++nt) {
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            pv[nt][e] = (g < p.G) ? exp2f(x[nt][e] - m_use) : 0.f;
                            psum += pv[nt][e];
                        }
                    }
                    l_run = l_run * alpha + psum;
                    m_run = m_new;
#pragma unroll
                    for (int dt = 0; dt < C::kDTiles; ++dt) {
                        o[dt][0] *= alpha;
                        o[dt][1] *= alpha;
                    }
                    // ---- zero V rows past the sequence end inside this warp's slice
                    if (valid < tbase + C::kTokPerWarp) {
                        const int first_bad = valid;
                        const int nrows = tbase + C::kTokPerWarp - first_bad;
                        for (int idx = lane; idx < nrows * C::kBoxes * 8; idx += 32) {
                            const int row = first_bad + idx / (C::kBoxes * 8);
                            const int rem = idx % (C::kBoxes * 8);
                            const uint32_t a = stV + (rem >> 3) * C::kBoxBytes + row * 128 + (rem & 7) * 16;
                            asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(0u) : "memory");
                        }
                        wrote = true;
                        __syncwarp();
                    }
                    // ---- O += P V (rows: heads, cols: head_dim)
                    if constexpr (C::kNT8 == 1) {
                        const uint32_t a0 = pack_bf16x2(pv[0][0], pv[0][1]);
                        const int mi = lane >> 3;
                        const int tok = tbase + (lane & 7);
#pragma unroll
                        for (int dq = 0; dq < C::kDTiles / 4; ++dq) {
                            uint32_t b[4];
                            ldmatrix_x4_trans(swz<BLK>(stV, tok, (dq * 4 + mi) * 8), b[0], b[1], b[2], b[3]);
#pragma unroll
                            for (int u = 0; u < 4; ++u) mma_bf16_1688(o[dq * 4 + u], a0, 0u, b[u]);
                        }
                    } else {
                        const uint32_t a0 = pack_bf16x2(pv[0][0], pv[0][1]);
                        const uint32_t a2 = pack_bf16x2(pv[1][0], pv[1][1]);
                        const int mi = lane >> 3;
                        const int tok = tbase + (mi & 1) * 8 + (lane & 7);
#pragma unroll
                        for (int dp = 0; dp < C::kDTiles / 2; ++dp) {
                            uint32_t b0, b1, b2, b3;
                            ldmatrix_x4_trans(swz<BLK>(stV, tok, (2 * dp + (mi >> 1)) * 8), b0, b1, b2, b3);
                            mma_bf16_16816(o[2 * dp], a0, 0u, a2, 0u, b0, b1);
                            mma_bf16_16816(o[2 * dp + 1], a0, 0u, a2, 0u, b2, b3);
                        }
                    }
                }
                if (wrote) fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_empty(st));
                if (++st == p.nst) {
                    st = 0;
                    ph ^= 1u;
                }
            }
            if (!ok) {
                if (ctid < p.G) p.lse_part[(head0 + ctid) * p.S + s.slot] = NAN;
                break;
            }

            // ---- merge the eight warp states of this segment into its slot
            l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
            l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
            if (g < p.G) {
                if (tig == 0) {
                    mM[warp * p.G + g] = m_run;
                    mL[warp * p.G + g] = l_run;
                }
                float* dst = mO + (size_t)(warp * p.G + g) * D + 2 * tig;
#pragma unroll
                for (int dt = 0; dt < C::kDTiles; ++dt)
                    *reinterpret_cast<float2*>(dst + dt * 8) = make_float2(o[dt][0], o[dt][1]);
            }
            mbar_arrive(bar_cons);
            if (!mbar_wait(bar_cons, cph)) {
                record_failure(abort_flag);
                ok = false;
            }
            cph ^= 1u;
            if (ok) {
                for (int idx = ctid; idx < p.G * D; idx += kConsumerThreads) {
                    const int h = idx / D, d = idx - h * D;
                    float M = -INFINITY;
#pragma unroll
                    for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, mM[w * p.G + h]);
                    float* lse_dst = p.lse_part + (head0 + h) * p.S + s.slot;
                    if (M == -INFINITY) {
                        if (d == 0) *lse_dst = -INFINITY;
                        continue;
                    }
                    float wsum = 0.f, acc = 0.f;
#pragma unroll
                    for (int w = 0; w < kConsumerWarps; ++w) {
                        const float mw = mM[w * p.G + h];
                        if (mw != -INFINITY) {
                            const float e = exp2f(mw - M);
                            wsum += e * mL[w * p.G + h];
                            acc += e * mO[(size_t)(w * p.G + h) * D + d];
                        }
                    }
                    p.o_part[((head0 + h) * p.S + s.slot) * D + d] = acc / wsum;
                    if (d == 0) *lse_dst = (M + log2f(wsum)) * kLn2;
                }
                // the merge area is reused by the next segment
                mbar_arrive(bar_cons);
                if (!mbar_wait(bar_cons, cph)) {
                    record_failure(abort_flag);
                    ok = false;
                }
                cph ^= 1u;
            }
        } else if (ctid < p.G) {
            p.lse_part[(head0 + ctid) * p.S + s.slot] = -INFINITY;  // no kept block in this piece
        }
        if (s.last) {
            const int rest = p.S - s.nslots;
            for (int idx = ctid; idx < p.G * rest; idx += kConsumerThreads) {
                const int h = idx / rest;
                p.lse_part[(head0 + h) * p.S + s.nslots + (idx - h * rest)] = -INFINITY;
            }
        }
    }
}

struct Layout {
    int nst, stage_bytes, merge_off, info_off, bar_off, total;
};

template <int D, int BLK>
Layout make_layout(int G) {
    using C = Cfg<D, BLK>;
    Layout l;
    l.stage_bytes = (2 * C::kTileBytes + G * D * 2 + 1023) / 1024 * 1024;
    const int merge_bytes = kConsumerWarps * G * D * 4 + 2 * kConsumerWarps * G * 4;
    const int tail = merge_bytes + (kMaxStages + 4) * 4 + (2 * kMaxStages + 2) * 8 + 64;
    int nst = (kSmemLimit - 1024 - tail) / l.stage_bytes;
    l.nst = nst > kMaxStages ? kMaxStages : nst;
    l.merge_off = l.nst * l.stage_bytes;
    l.info_off = (l.merge_off + merge_bytes + 15) / 16 * 16;
    l.bar_off = (l.info_off + (kMaxStages + 4) * 4 + 15) / 16 * 16;
    l.total = l.bar_off + (2 * l.nst + 2) * 8 + 1024;  // + slack for the 1024-byte alignment
    return l;
}

template <int D, int BLK>
cudaError_t launch_impl(const Shape& s, const DecodeLaunch& a, const CUtensorMap& tmK, const CUtensorMap& tmV,
                        int num_sms, cudaStream_t stream) {
    const Layout l = make_layout<D, BLK>(s.G);
    if (l.nst < 2) return cudaErrorInvalidConfiguration;
    static bool attr_done = false;  // set once per template instance (benign race)
    if (!attr_done) {
        cudaError_t e =
            cudaFuncSetAttribute(sparse_decode_kernel<D, BLK>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit);
        if (e != cudaSuccess) return e;
        attr_done = true;
    }
    Params p;
    p.q = static_cast<const __nv_bfloat16*>(a.q);
    p.seq_lens = a.seq_lens;
    p.block_idx = a.block_idx;
    p.num_selected = a.num_selected;
    p.o_part = a.o_part;
    p.lse_part = a.lse_part;
    p.V = (long long)s.B * s.Hkv * a.kmax;
    p.Hq = s.Hq;
    p.Hkv = s.Hkv;
    p.G = s.G;
    p.Lmax = s.Lmax;
    p.kmax = a.kmax;
    p.S = a.num_splits;
    p.P = sparse_decode_ctas(s, a.kmax, a.num_splits, num_sms);
    p.nst = l.nst;
    p.stage_bytes = l.stage_bytes;
    p.merge_off = l.merge_off;
    p.info_off = l.info_off;
    p.bar_off = l.bar_off;
    p.scale_log2 = a.sm_scale * kLog2e;
    sparse_decode_kernel<D, BLK><<<p.P, kThreads, l.total, stream>>>(tmK, tmV, p);
    return cudaGetLastError();
}

}  // namespace

int sparse_decode_ctas(const Shape& s, int kmax, int num_splits, int num_sms) {
    const long long V = (long long)s.B * s.Hkv * kmax;
    const int full = kmax < num_sms ? kmax : num_sms;
    long long P = (num_splits >= full) ? num_sms : num_splits;
    if (P > V) P = V;
    return P < 1 ? 1 : (int)P;
}

cudaError_t launch_sparse_decode(const Shape& s, const DecodeLaunch& a, const CUtensorMap& tmK,
                                 const CUtensorMap& tmV, int num_sms, cudaStream_t stream) {
    if (s.D == 128 && s.blk == 64) return launch_impl<128, 64>(s, a, tmK, tmV, num_sms, stream);
    if (s.D == 128 && s.blk == 128) return launch_impl<128, 128>(s, a, tmK, tmV, num_sms, stream);
    if (s.D == 64 && s.blk == 64) return launch_impl<64, 64>(s, a, tmK, tmV, num_sms, stream);
    if (s.D == 64 && s.blk == 128) return launch_impl<64, 128>(s, a, tmK, tmV, num_sms, stream);
    return cudaErrorInvalidValue;
}

}  // namespace seer
