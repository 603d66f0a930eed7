// sparse_decode.cu -- block-sparse split-KV flash-decode for sm_100a, and the
// whole decode step fused into one cooperative launch.
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
//    produces one partial (o, lse) "slot".
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
//  * every wait is bounded (mbarrier waits and the grid barrier alike); on
//    expiry the CTA counts a failure, writes NaN into the slot it was
//    producing and leaves only after its own copies have landed.
//
// sparse_decode_kernel (seer_sparse_decode) writes the slots; seer_combine
// merges them. decode_step_kernel (seer_decode_step) runs the whole step in
// one cooperative launch:
//   phase 1, one CTA per row (strided): refresh the pooled-K rows of the open
//     block(s), project the group's mean query, score the cached pooled keys
//     (streamed into the idle stage ring by bulk copies), select the kept
//     blocks -- with the same arithmetic as the separate kernels
//     (gate_core.cuh), so both paths give bit-identical block lists;
//   a bounded grid barrier;
//   phase 2, the decode above; the last CTA to finish a row's slots (an
//     atomic count per row) merges them into the output in place of
//     seer_combine, and resets the count for the next call.
#include <cfloat>
#include <cmath>

#include "gate_core.cuh"
#include "seer_launch.h"

namespace seer {

// Count of CTAs that gave up on a bounded wait (0 in normal operation).
__device__ unsigned int g_decode_wait_failures = 0;

namespace {

constexpr int kConsumerWarps = 8;
constexpr int kConsumerThreads = kConsumerWarps * 32;
constexpr int kThreads = kConsumerThreads + 32;       // standalone decode: consumers + producer
constexpr int kHelperWarp0 = kConsumerWarps + 1;       // fused step: + 3 helper warps
constexpr int kHelperThreads = 96;
constexpr int kStepThreads = kThreads + kHelperThreads;  // 12 warps: the register budget of 9 (allocated as 12)
constexpr int kMaxStages = 8;
constexpr int kMaxGateStages = 8;
constexpr int kSmemLimit = 232448;       // 227 KB of opt-in dynamic shared memory per CTA
constexpr int kGateScratchBytes = 16384;  // phase-1 scratch at the start of the stage ring
constexpr int kGateChunkBytes = 32768;    // phase-1 bulk copy unit (pooled-K rows)
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

// Extra arguments of the fused step (phase 1 and the in-kernel merge).
struct StepParams {
    const __nv_bfloat16* k_cache;
    const float* w_q;
    const float* w_k;
    const int32_t* upd_start;
    float* kpool;
    int32_t* block_idx;     // phase-1 output, phase-2 input
    int32_t* num_selected;  // idem
    __nv_bfloat16* out;
    float* lse_out;
    unsigned int* grid_bar;  // 64-bit arrival counter (grows by gridDim.x per launch)
    unsigned int* row_done;  // [rows] finished decode slots per row
    unsigned int* row_cnt;   // [rows] finished phase-1 pieces per row
    unsigned int* qg_flag;   // [rows] the row's projected query is in qg_g
    float* qg_g;             // [rows, dg] projected queries, written by each row's first CTA
    uint32_t* keys_g;        // [rows, NBmax] order keys of the block scores
    int rows, NBmax, dg;
    int gate_ctas;                           // CTAs of phase 1 (a multiple of rows when rows fit the grid)
    int keys_off, chunk_off, n_gate_stages;  // phase-1 layout inside the stage ring
    int refresh_off;                         // phase-2 pool scratch (outside the ring)
};

// Shared-memory info words after the per-stage `valid` counts.
constexpr int kInfoAbort = kMaxStages;      // a wait of this CTA gave up
constexpr int kInfoMergeRow = kMaxStages + 1;  // this CTA merges the current row
constexpr int kInfoWords = kMaxStages + 4;

// One row's share of this CTA's range.
struct Segment {
    int row, b, kvh, L, a0, a1, slot, nslots;
    bool last;  // this CTA holds the end of the row's reserved positions
};

template <bool kFresh>
__device__ __forceinline__ int load_i32(const int32_t* p) {
    // Values written earlier in the same launch by other CTAs bypass L1.
    if constexpr (kFresh) return __ldcg(p);
    else return *p;
}

template <bool kFused>
__device__ __forceinline__ Segment make_segment(const Params& p, int r, long long g0, long long g1) {
    Segment s;
    const long long rs = (long long)r * p.kmax;
    const int i0 = (int)(g0 > rs ? g0 - rs : 0);
    const int i1 = (int)((g1 - rs) < p.kmax ? (g1 - rs) : p.kmax);
    s.row = r;
    s.b = r / p.Hkv;
    s.kvh = r - s.b * p.Hkv;
    s.L = clamp_len(p.seq_lens[s.b], p.Lmax);
    int n = s.L == 0 ? 0 : load_i32<kFused>(p.num_selected + r);
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

__device__ __forceinline__ void record_failure(int* info) {
    if (atomicExch(info + kInfoAbort, 1) == 0) atomicAdd(&g_decode_wait_failures, 1u);
}

// Shared-memory views common to both kernels.
struct Smem {
    unsigned char* base;  // 1024-aligned
    uint32_t sbase;
    float* merge;
    int* info;
    uint32_t bars;
    int nst;
    __device__ __forceinline__ uint32_t full(int st) const { return bars + 8u * st; }
    __device__ __forceinline__ uint32_t empty(int st) const { return bars + 8u * (nst + st); }
    __device__ __forceinline__ uint32_t cons() const { return bars + 16u * nst; }
    __device__ __forceinline__ uint32_t gate(int st) const { return bars + 16u * nst + 8u + 8u * st; }
    __device__ __forceinline__ uint32_t helper() const { return bars + 16u * nst + 8u + 8u * kMaxGateStages; }
};

__device__ __forceinline__ Smem setup_smem(unsigned char* raw, const Params& p) {
    Smem m;
    m.base = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
    m.sbase = smem_addr(m.base);
    m.merge = reinterpret_cast<float*>(m.base + p.merge_off);
    m.info = reinterpret_cast<int*>(m.base + p.info_off);
    m.bars = m.sbase + p.bar_off;
    m.nst = p.nst;
    if (threadIdx.x == 0) {
        for (int st = 0; st < p.nst; ++st) {
            mbar_init(m.full(st), 1);
            mbar_init(m.empty(st), kConsumerWarps);
        }
        mbar_init(m.cons(), kConsumerThreads);
        for (int st = 0; st < kMaxGateStages; ++st) mbar_init(m.gate(st), 1);
        mbar_init(m.helper(), kHelperThreads);
        for (int i = 0; i < kInfoWords; ++i) m.info[i] = 0;
        fence_mbar_init();
    }
    __syncthreads();
    return m;
}

// All 256 consumer threads meet (bounded); false if the wait gave up.
__device__ __forceinline__ bool consumer_sync(const Smem& m, uint32_t& cph) {
    mbar_arrive(m.cons());
    const bool ok = mbar_wait(m.cons(), cph);
    cph ^= 1u;
    if (!ok) record_failure(m.info);
    return ok;
}

// ---------------------------------------------------------------- decode: producer warp

template <int D, int BLK, bool kFused>
__device__ void decode_producer(const CUtensorMap* tmK, const CUtensorMap* tmV, const Params& p, const Smem& m,
                                long long g0, long long g1) {
    using C = Cfg<D, BLK>;
    const int lane = threadIdx.x & 31;
    if (lane == 0) {
        prefetch_tensor_map(tmK);
        prefetch_tensor_map(tmV);
    }
    const uint64_t policy = l2_policy_evict_first();
    int st = 0;
    uint32_t ph = 0;
    long long issued = 0;
    bool ok = true;
    for (int r = (int)(g0 / p.kmax); ok && (long long)r * p.kmax < g1; ++r) {
        const Segment s = make_segment<kFused>(p, r, g0, g1);
        if (s.a1 <= s.a0) continue;
        const int NB = (s.L + BLK - 1) / BLK;
        const __nv_bfloat16* qsrc = p.q + ((size_t)s.b * p.Hq + (size_t)s.kvh * p.G) * D;
        const int32_t* list = p.block_idx + (size_t)r * p.kmax;
        for (int i = s.a0; ok && i < s.a1; i += 32) {
            const int jl = (i + lane < s.a1) ? load_i32<kFused>(list + i + lane) : -1;
            const int cnt = min(32, s.a1 - i);
            for (int k = 0; ok && k < cnt; ++k) {
                const int j = __shfl_sync(0xffffffffu, jl, k);
                const int valid = (j >= 0 && j < NB) ? min(BLK, s.L - j * BLK) : 0;
                int good = 1;
                if (lane == 0) {
                    if (!mbar_wait(m.empty(st), ph ^ 1u)) {
                        good = 0;
                        record_failure(m.info);
                    } else {
                        m.info[st] = valid;
                        const bool first = (i + k == s.a0);
                        const uint32_t fb = m.full(st);
                        const uint32_t bytes =
                            (valid > 0 ? 2u * C::kTileBytes : 0u) + (first ? (uint32_t)(p.G * D * 2) : 0u);
                        if (bytes) mbar_arrive_expect_tx(fb, bytes);
                        else mbar_arrive(fb);
                        const uint32_t stK = m.sbase + (uint32_t)st * p.stage_bytes;
                        if (valid > 0) {
                            const int y = r * p.Lmax + j * BLK;
#pragma unroll
                            for (int bx = 0; bx < C::kBoxes; ++bx) {
                                tma_load_2d(stK + bx * C::kBoxBytes, tmK, fb, bx * 64, y, policy);
                                tma_load_2d(stK + C::kTileBytes + bx * C::kBoxBytes, tmV, fb, bx * 64, y, policy);
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
            if (!ok || !mbar_wait(m.empty(s_it), par)) (void)mbar_wait(m.full(s_it), par);
        }
    }
}

// ---------------------------------------------------------------- decode: in-kernel merge (fused step)

// The last CTA to finish a slot of row `s.row` merges all of the row's slots
// into out / lse_out (log-sum-exp weights) and resets the row's count.
template <int D>
__device__ void merge_row_if_last(const Params& p, const StepParams& f, const Smem& m, const Segment& s,
                                  uint32_t& cph) {
    const int ctid = threadIdx.x;
    if (!consumer_sync(m, cph)) return;  // the CTA's slot writes, then its release-add
    if (ctid == 0) {
        const unsigned int done = atomic_add_acq_rel(f.row_done + s.row, 1u) + 1u;
        m.info[kInfoMergeRow] = (done == (unsigned int)s.nslots);
    }
    if (!consumer_sync(m, cph)) return;  // the acquire, then every consumer reads the slots
    if (!m.info[kInfoMergeRow]) return;
    const size_t head0 = (size_t)s.b * p.Hq + (size_t)s.kvh * p.G;
    const int ns = s.nslots;
    float* w = m.merge;  // [G][ns] normalised slot weights (the merge area is free here)
    if (ctid < p.G) {
        const float* l = p.lse_part + (head0 + ctid) * p.S;
        float M = -INFINITY;
        for (int k = 0; k < ns; ++k) M = fmaxf(M, __ldcg(l + k));
        float wsum = 0.f;
        for (int k = 0; k < ns; ++k) {
            const float lk = __ldcg(l + k);
            const float e = (lk == -INFINITY || M == -INFINITY) ? 0.f : expf(lk - M);
            w[ctid * ns + k] = e;
            wsum += e;
        }
        const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
        for (int k = 0; k < ns; ++k) w[ctid * ns + k] *= inv;
        if (f.lse_out) f.lse_out[head0 + ctid] = (M == -INFINITY) ? -INFINITY : M + logf(wsum);
    }
    if (!consumer_sync(m, cph)) return;
    for (int idx = ctid; idx < p.G * D; idx += kConsumerThreads) {
        const int h = idx / D, d = idx - h * D;
        float acc = 0.f;
        for (int k = 0; k < ns; ++k) {
            const float wk = w[h * ns + k];
            if (wk != 0.f) acc += wk * __ldcg(p.o_part + ((head0 + h) * p.S + k) * D + d);
        }
        f.out[(head0 + h) * D + d] = __float2bfloat16(acc);
    }
    if (ctid == 0) f.row_done[s.row] = 0u;
    (void)consumer_sync(m, cph);  // the weights area is reused by the next segment
}

// ---------------------------------------------------------------- decode: consumer warps

template <int D, int BLK, bool kFused>
__device__ void decode_consumers(const Params& p, const StepParams& f, const Smem& m, long long g0, long long g1) {
    using C = Cfg<D, BLK>;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ctid = threadIdx.x;                  // 0 .. 255
    const int g = lane >> 2, tig = lane & 3;       // mma fragment coordinates
    const int tbase = warp * C::kTokPerWarp;       // this warp's token slice of each block
    float* mO = m.merge;                           // [8][G][D]
    float* mM = m.merge + kConsumerWarps * p.G * D;  // [8][G]
    float* mL = mM + kConsumerWarps * p.G;         // [8][G]
    int st = 0;
    uint32_t ph = 0, cph = 0;
    bool ok = true;

    for (int r = (int)(g0 / p.kmax); ok && (long long)r * p.kmax < g1; ++r) {
        const Segment s = make_segment<kFused>(p, r, g0, g1);
        const size_t head0 = (size_t)s.b * p.Hq + (size_t)s.kvh * p.G;
        if (s.a1 > s.a0) {
            float m_run = -INFINITY, l_run = 0.f;
            float o[C::kDTiles][4];
#pragma unroll
            for (int dt = 0; dt < C::kDTiles; ++dt) o[dt][0] = o[dt][1] = o[dt][2] = o[dt][3] = 0.f;
            uint32_t qa[C::kKSteps][2];

            for (int i = s.a0; i < s.a1; ++i) {
                if (!mbar_wait(m.full(st), ph)) {
                    record_failure(m.info);
                    ok = false;
                    break;
                }
                const int valid = m.info[st];
                const uint32_t stK = m.sbase + (uint32_t)st * p.stage_bytes;
                const uint32_t stV = stK + C::kTileBytes;
                if (i == s.a0) {
                    const __nv_bfloat16* qs = reinterpret_cast<const __nv_bfloat16*>(
                        m.base + (size_t)st * p.stage_bytes + 2 * C::kTileBytes);
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
                if (lane == 0) mbar_arrive(m.empty(st));
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
            if (!(ok = consumer_sync(m, cph))) break;
            for (int idx = ctid; idx < p.G * D; idx += kConsumerThreads) {
                const int h = idx / D, d = idx - h * D;
                float M = -INFINITY;
#pragma unroll
                for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, mM[w * p.G + h]);
                float* lse_dst = p.lse_part + (head0 + h) * p.S + s.slot;
                const bool direct = kFused && s.nslots == 1;  // the row's only piece: straight to the output
                if (M == -INFINITY) {
                    if (direct) {
                        f.out[(head0 + h) * D + d] = __float2bfloat16(0.f);
                        if (d == 0 && f.lse_out) f.lse_out[head0 + h] = -INFINITY;
                    } else if (d == 0) {
                        *lse_dst = -INFINITY;
                    }
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
                if (direct) {
                    f.out[(head0 + h) * D + d] = __float2bfloat16(acc / wsum);
                    if (d == 0 && f.lse_out) f.lse_out[head0 + h] = (M + log2f(wsum)) * kLn2;
                    continue;
                }
                p.o_part[((head0 + h) * p.S + s.slot) * D + d] = acc / wsum;
                if (d == 0) *lse_dst = (M + log2f(wsum)) * kLn2;
            }
            // the merge area is reused by the next segment
            if (!(ok = consumer_sync(m, cph))) break;
        } else if (kFused && s.nslots == 1) {  // a row without tokens, in one piece
            for (int idx = ctid; idx < p.G * D; idx += kConsumerThreads)
                f.out[head0 * D + idx] = __float2bfloat16(0.f);
            if (ctid < p.G && f.lse_out) f.lse_out[head0 + ctid] = -INFINITY;
        } else if (ctid < p.G) {
            p.lse_part[(head0 + ctid) * p.S + s.slot] = -INFINITY;  // no kept block in this piece
        }
        if constexpr (kFused) {
            if (s.nslots > 1) merge_row_if_last<D>(p, f, m, s, cph);  // else written above
            ok = m.info[kInfoAbort] == 0;
        } else if (s.last) {
            const int rest = p.S - s.nslots;
            for (int idx = ctid; idx < p.G * rest; idx += kConsumerThreads) {
                const int h = idx / rest;
                p.lse_part[(head0 + h) * p.S + s.nslots + (idx - h * rest)] = -INFINITY;
            }
        }
    }
}

// ---------------------------------------------------------------- fused step: helper warps

// First block to refresh for sequence b (upd_start, by default the token just appended).
__device__ __forceinline__ int refresh_start_block(const StepParams& f, int b, int L, int NB, int blk) {
    int st0 = f.upd_start ? f.upd_start[b] : L - 1;
    st0 = st0 < 0 ? 0 : st0;
    return min(st0 / blk, NB);
}

// Phase 2, warps 9..11, beside the decode: refresh the pooled key of the open
// last block of every row whose first slot this CTA holds. Phase 1 never reads
// it (the last block is always kept), so it runs while the decode streams.
template <int D, int BLK>
__device__ void decode_helpers(const Params& p, const StepParams& f, const Smem& m, long long g0, long long g1) {
    PoolSmem<D>& psm = *reinterpret_cast<PoolSmem<D>*>(m.base + f.refresh_off);
    const int hwarp = ((int)threadIdx.x >> 5) - kHelperWarp0, lane = threadIdx.x & 31;
    uint32_t hph = 0;
    bool ok = true;
    auto hsync = [&]() {
        if (!ok) return;
        mbar_arrive(m.helper());
        ok = mbar_wait(m.helper(), hph);
        hph ^= 1u;
        if (!ok) record_failure(m.info);
    };
    for (int r = (int)(g0 / p.kmax); ok && (long long)r * p.kmax < g1; ++r) {
        const Segment s = make_segment<true>(p, r, g0, g1);
        if (s.slot != 0 || s.L == 0) continue;
        const int NB = (s.L + BLK - 1) / BLK;
        if (refresh_start_block(f, s.b, s.L, NB, BLK) > NB - 1) continue;
        const int j = NB - 1;
        pool_block_mean<D, BLK>(f.k_cache + ((size_t)r * p.Lmax + (size_t)j * BLK) * D, s.L - j * BLK, psm, hsync,
                                kHelperWarp0 * 32);
        float pv[D / 32];
#pragma unroll
        for (int u = 0; u < D / 32; ++u) pv[u] = psm.pooled[lane * (D / 32) + u];
        float* dst = f.kpool + ((size_t)r * f.NBmax + j) * f.dg;
        const float* W = f.w_k + (size_t)s.kvh * f.dg * D;
        warp_matvec_rows<D>(W, pv, hwarp, f.dg, kHelperThreads / 32, [&](int e, float x) { dst[e] = x; });
        hsync();  // the pool scratch is reused by the next row
    }
}

template <int D, int BLK>
__global__ void __launch_bounds__(kThreads, 1)  // 9 warps are allocated registers as 12: <= 168 each
    sparse_decode_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                         const Params p) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const Smem m = setup_smem(smem_raw, p);
    const long long g0 = (long long)blockIdx.x * p.V / p.P;
    const long long g1 = (long long)(blockIdx.x + 1) * p.V / p.P;
    if ((threadIdx.x >> 5) == kConsumerWarps) decode_producer<D, BLK, false>(&tmK, &tmV, p, m, g0, g1);
    else decode_consumers<D, BLK, false>(p, StepParams{}, m, g0, g1);
}

// ---------------------------------------------------------------- fused step: phase 1 (gate + select)

// One row of the rows a CTA meets in its phase-1 range.
struct GateRow {
    int r, b, kvh, L, NB, js;  // js: first block whose pooled key is refreshed
    int s0, s1;                // cached positions [s0, s1) this CTA scores
    int scored;                // the row's choice needs scores
    int refresh_now;           // this CTA refreshes the competing blocks [js, NB-1) here
};
constexpr int kMaxBatchRows = 8;

template <int D, int DG>
struct GateScratch {
    alignas(16) float qbar[kMaxBatchRows][D];
    alignas(16) float qg[kMaxBatchRows][DG];
    alignas(16) float kp_new[DG];
    PoolSmem<D> pool;
    GateRow rows[kMaxBatchRows];
    int last_of[kMaxBatchRows];
};
static_assert(sizeof(GateScratch<128, 128>) <= kGateScratchBytes, "phase-1 scratch");
static_assert(sizeof(SelectSmem<kStepThreads>) <= kGateChunkBytes, "the select scratch reuses a chunk stage");
static_assert(sizeof(GateScratch<64, 128>) <= kGateScratchBytes, "phase-1 scratch");

// Phase 1. The R x NBmax pooled-key positions (row-major, the layout of
// kpool) are cut into gridDim.x equal contiguous ranges. Each CTA streams the
// cached rows of its range into the stage ring (bulk copies), scores them
// against the projected query of their row (a lane quad per row), and writes
// order keys to the workspace. A per-row count of finished ranges tells the
// last CTA of a row to run that row's selection. The open last block is never
// a candidate, so its pooled key is refreshed in phase 2; only blocks that
// compete (a refresh point before the last block) are refreshed here.
template <int D, int BLK, int DG>
__device__ void gate_phase(const Params& p, const StepParams& f, const Smem& m) {
    constexpr int kThreads = kStepThreads;
    constexpr int kWarps = kThreads / 32;
    constexpr int kChunkRows = kGateChunkBytes / (DG * 4);
    constexpr int kVecD = D / 32;
    using WVec = typename std::conditional<kVecD == 4, float4, float2>::type;
    GateScratch<D, DG>& sm = *reinterpret_cast<GateScratch<D, DG>*>(m.base);
    uint32_t* keys = reinterpret_cast<uint32_t*>(m.base + f.keys_off);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = lane >> 2, qlane = lane & 3;
    const float inv_sqrt_dg = 1.0f / sqrtf((float)DG);
    const long long V1 = (long long)f.rows * f.NBmax;
    // With no more rows than CTAs each row goes to the same whole number of
    // CTAs (one CTA per row needs no hand-offs: its keys stay in shared memory
    // and it selects right after scoring); with more rows the positions are
    // spread evenly over every CTA.
    const int G1 = f.gate_ctas;
    if ((int)blockIdx.x >= G1) return;
    const long long h0 = (long long)blockIdx.x * V1 / G1;
    const long long h1 = (long long)(blockIdx.x + 1) * V1 / G1;
    const bool whole_rows = G1 == f.rows;
    // Rows r with r * NBmax < h1, from the row holding h0: exactly the rows
    // whose [first, last] covering-CTA interval contains this CTA (an empty
    // range strictly inside a row still counts for that row).
    const int r_stop = (int)((h1 + f.NBmax - 1) / f.NBmax);
    int chunk_it = 0;  // bulk copies consumed so far (the same count on every thread)

    for (int r = (int)(h0 / f.NBmax); r < r_stop;) {
        const int nb = min(kMaxBatchRows, r_stop - r);
        // ---- (1) before anything else reaches DRAM: the projection weights of the
        //      batch rows (first kQBatch outputs per warp), their lengths and
        //      group-mean queries -- all independent loads, issued together
        constexpr int kQBatch = 16;
        // A row's first position lies in exactly one CTA's range: that CTA owns
        // the row and projects its query; the owned rows of a batch are contiguous.
        auto owner_of = [&](int row) {
            const long long x = (long long)row * f.NBmax;
            return x >= h0 && x < h1;
        };
        int own_first = nb, own_rows = 0;
        for (int k = 0; k < nb; ++k)
            if (owner_of(r + k)) {
                own_first = min(own_first, k);
                ++own_rows;
            }
        const int total_q = own_rows * DG;  // outputs ordered by owned row, then e
        auto owned_row = [&](int o) { return own_first + o / DG; };
        // lengths and update starts of the batch rows: independent loads, issued first
        int len_raw = 0, upd_raw = -1;
        if (tid < nb) {
            const int b = (r + tid) / p.Hkv;
            len_raw = load_early(p.seq_lens + b);
            if (f.upd_start) upd_raw = load_early(f.upd_start + b);
        }
        WVec w[kQBatch];
        if (total_q > 0) {
#pragma unroll
            for (int u = 0; u < kQBatch; ++u) {
                const int o = min(warp + u * kWarps, total_q - 1);
                const int k = owned_row(o), e = o % DG;
                const int kvh = (r + k) % p.Hkv;
                load_early(w[u], f.w_q + ((size_t)kvh * DG + e) * D + lane * kVecD);
            }
        }

        if (tid < nb) {
            GateRow& g = sm.rows[tid];
            g.r = r + tid;
            g.b = g.r / p.Hkv;
            g.kvh = g.r - g.b * p.Hkv;
            g.L = clamp_len(len_raw, p.Lmax);
            g.NB = (g.L + BLK - 1) / BLK;
            const int st0 = max(f.upd_start ? upd_raw : g.L - 1, 0);  // as refresh_start_block
            g.js = g.NB > 0 ? min(st0 / BLK, g.NB) : g.NB;
        }
        for (int idx = tid; idx < nb * D; idx += kThreads) {
            const int k = idx / D, d = idx - k * D;
            const int row = r + k, b = row / p.Hkv, kvh = row - b * p.Hkv;
            if (owner_of(row))
                sm.qbar[k][d] = group_query_mean_at(p.q + ((size_t)b * p.Hq + (size_t)kvh * p.G) * D, p.G, D, d);
        }
        __syncthreads();
        if (tid < nb) {
            GateRow& g = sm.rows[tid];
            const long long rs = (long long)g.r * f.NBmax;
            const int i0 = (int)(h0 > rs ? h0 - rs : 0);
            const int i1 = (int)((h1 - rs) < f.NBmax ? (h1 - rs) : f.NBmax);
            const int kb = p.kmax < g.NB ? p.kmax : g.NB;
            const int ncand = g.NB - 1;
            g.scored = kb - 1 > 0 && kb - 1 < ncand;
            const int lim = g.scored ? min(g.js, ncand) : 0;
            g.s0 = min(i0, lim);
            g.s1 = min(i1, lim);
            g.refresh_now = g.js < ncand && g.js >= i0 && g.js < i1;
        }
        __syncthreads();
        auto nchunks_of = [&](int k) { return (sm.rows[k].s1 - sm.rows[k].s0 + kChunkRows - 1) / kChunkRows; };
        int total_chunks = 0;
        for (int k = 0; k < nb; ++k) total_chunks += nchunks_of(k);
        auto chunk = [&](int i, int& k, int& j0, int& n) {
            for (k = 0; k < nb - 1; ++k) {
                const int c = nchunks_of(k);
                if (i < c) break;
                i -= c;
            }
            j0 = sm.rows[k].s0 + i * kChunkRows;
            n = min(kChunkRows, sm.rows[k].s1 - j0);
        };
        auto issue = [&](int i) {
            int k, j0, n;
            chunk(i, k, j0, n);
            const int stage = (chunk_it + i) % f.n_gate_stages;
            const uint32_t bytes = (uint32_t)(n * DG * 4);
            mbar_arrive_expect_tx(m.gate(stage), bytes);
            bulk_load(m.sbase + (uint32_t)(f.chunk_off + stage * kGateChunkBytes),
                      f.kpool + ((size_t)sm.rows[k].r * f.NBmax + j0) * DG, bytes, m.gate(stage));
        };
        // ---- (2) stream the cached pooled keys; meanwhile project the owned rows' queries
        if (tid == 0)
            for (int i = 0; i < min(f.n_gate_stages, total_chunks); ++i) issue(i);
        if (total_q > 0) {
#pragma unroll
            for (int u = 0; u < kQBatch; ++u) {
                const int o = warp + u * kWarps;
                const int oc = min(o, total_q - 1);
                const int k = owned_row(oc), e = oc % DG;
                const float x = warp_sum(piece_dot(w[u], &sm.qbar[k][lane * kVecD]));
                if (lane == 0 && o < total_q) sm.qg[k][e] = x;
            }
            for (int o0 = warp + kQBatch * kWarps; o0 < total_q; o0 += 8 * kWarps) {  // batches beyond the first
                WVec w2[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int o = min(o0 + u * kWarps, total_q - 1);
                    const int k = owned_row(o), e = o % DG;
                    w2[u] = *reinterpret_cast<const WVec*>(f.w_q + ((size_t)sm.rows[k].kvh * DG + e) * D + lane * kVecD);
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int o = o0 + u * kWarps;
                    const int oc = min(o, total_q - 1);
                    const int k = owned_row(oc), e = oc % DG;
                    const float x = warp_sum(piece_dot(w2[u], &sm.qbar[k][lane * kVecD]));
                    if (lane == 0 && o < total_q) sm.qg[k][e] = x;
                }
            }
        }
        __syncthreads();
        // publish every owned projection first, then fetch the others' (their owners are
        // lower-indexed CTAs that publish before they wait on anyone: no chains)
        if (!whole_rows) {
            for (int k = 0; k < nb; ++k)
                if (owner_of(sm.rows[k].r) && sm.rows[k].scored)
                    for (int e = tid; e < DG; e += kThreads) f.qg_g[(size_t)sm.rows[k].r * DG + e] = sm.qg[k][e];
            __syncthreads();
            if (tid < nb && owner_of(sm.rows[tid].r) && sm.rows[tid].scored)
                asm volatile("st.release.gpu.u32 [%0], %1;" ::"l"(f.qg_flag + sm.rows[tid].r), "r"(1u) : "memory");
        }
        for (int k = 0; k < nb; ++k) {
            const GateRow& g = sm.rows[k];
            const bool needed = g.scored && (g.s1 > g.s0 || g.refresh_now);
            if (!owner_of(g.r) && needed) {
                if (tid == 0) {
                    const uint64_t t0 = global_timer_ns();
                    while (true) {
                        unsigned int v;
                        asm volatile("ld.acquire.gpu.u32 %0, [%1];" : "=r"(v) : "l"(f.qg_flag + g.r) : "memory");
                        if (v) break;
                        if (global_timer_ns() - t0 > kWaitLimitNs) {
                            record_failure(m.info);
                            break;
                        }
                        __nanosleep(128);
                    }
                }
                __syncthreads();
                for (int e = tid; e < DG; e += kThreads) sm.qg[k][e] = __ldcg(f.qg_g + (size_t)g.r * DG + e);
            }
        }
        __syncthreads();

        // ---- (3) refresh and score competing blocks of a refresh point inside the range (multi-token appends)
        for (int k = 0; k < nb; ++k) {
            const GateRow& g = sm.rows[k];
            if (!g.refresh_now) continue;
            const __nv_bfloat16* krow = f.k_cache + (size_t)g.r * p.Lmax * D;
            float* kp_row = f.kpool + (size_t)g.r * f.NBmax * DG;
            for (int j = g.js; j < g.NB - 1; ++j) {
                pool_block_mean<D, BLK>(krow + (size_t)j * BLK * D, min(BLK, g.L - j * BLK), sm.pool);
                float pv[kVecD];
#pragma unroll
                for (int u = 0; u < kVecD; ++u) pv[u] = sm.pool.pooled[lane * kVecD + u];
                warp_matvec_rows<D>(f.w_k + (size_t)g.kvh * DG * D, pv, warp, DG, kWarps, [&](int e, float x) {
                    kp_row[(size_t)j * DG + e] = x;
                    sm.kp_new[e] = x;
                });
                __syncthreads();
                if (warp == 0) {
                    const float d = quad_row_dot<DG>(sm.kp_new, j, sm.qg[k], qlane);
                    if (lane == 0)
                        (whole_rows ? keys : f.keys_g + (size_t)g.r * f.NBmax)[j] = order_key(d * inv_sqrt_dg);
                }
                __syncthreads();
            }
        }

        // ---- (4) score the cached rows as their copies land (a lane quad per row)
        for (int i = 0; i < total_chunks; ++i) {
            int k, j0, n;
            chunk(i, k, j0, n);
            const int stage = (chunk_it + i) % f.n_gate_stages;
            const uint32_t par = (uint32_t)(((chunk_it + i) / f.n_gate_stages) & 1);
            if (!mbar_wait(m.gate(stage), par)) record_failure(m.info);
            const float* tile = reinterpret_cast<const float*>(m.base + f.chunk_off + stage * kGateChunkBytes);
            uint32_t* kout = whole_rows ? keys : f.keys_g + (size_t)sm.rows[k].r * f.NBmax;
            const float* qg = sm.qg[k];
            for (int t0 = warp * 8; t0 < n; t0 += kWarps * 8) {
                const int t = min(t0 + quad, n - 1);
                const float d = quad_row_dot<DG>(tile + (size_t)t * DG, j0 + t, qg, qlane);
                if (qlane == 0 && t0 + quad < n) kout[j0 + t] = order_key(d * inv_sqrt_dg);
            }
            fence_proxy_async_smem();  // these generic reads of the stage precede its next bulk copy
            __syncthreads();
            if (tid == 0 && i + f.n_gate_stages < total_chunks) issue(i + f.n_gate_stages);
        }
        chunk_it += total_chunks;

        // ---- (5) count this CTA's pieces (one release-add per row, together);
        //      the last CTA of a row selects its blocks
        __syncthreads();  // every key of the batch written before the adds
        if (tid < nb) {
            const GateRow& g = sm.rows[tid];
            const long long rs = (long long)g.r * f.NBmax;
            if (whole_rows) {
                sm.last_of[tid] = 1;  // the only CTA of its row
            } else {
                const int cf = (int)(((rs + 1) * G1 - 1) / V1);
                const int cl = (int)(((rs + f.NBmax) * G1 - 1) / V1);
                const unsigned int done = atomic_add_acq_rel(f.row_cnt + g.r, 1u) + 1u;
                sm.last_of[tid] = done == (unsigned int)(cl - cf + 1);
            }
        }
        __syncthreads();
        // the rows this CTA completes: load their keys, then the CTA selects each
        SelectSmem<kThreads>& ssm = *reinterpret_cast<SelectSmem<kThreads>*>(m.base + f.chunk_off);
        for (int k = 0; k < nb; ++k) {
            if (!sm.last_of[k]) continue;
            const GateRow& g = sm.rows[k];
            if (g.scored && !whole_rows)
                for (int i = tid; i < g.NB - 1; i += kThreads) keys[i] = __ldcg(f.keys_g + (size_t)g.r * f.NBmax + i);
            if (tid == 0) {
                f.num_selected[g.r] = p.kmax < g.NB ? p.kmax : g.NB;
                f.row_cnt[g.r] = 0u;   // ready for the next call: every reader of the row's
                f.qg_flag[g.r] = 0u;   // projected query has counted in by now
            }
            __syncthreads();
            select_row<kThreads>(keys, g.NB, p.kmax, f.block_idx + (size_t)g.r * p.kmax, ssm);
            __syncthreads();
        }
        fence_proxy_async_smem();
        __syncthreads();  // scratch, keys and stages are reused by the next batch
        r += nb;
    }
}

// Bounded barrier over every CTA of a cooperative launch. One 64-bit arrival
// counter that only grows (every launch adds gridDim.x, from zero), so there
// is no reset step: a CTA's target is the next multiple of gridDim.x above
// the count it finds when it arrives, and the critical path is one atomic of
// the last CTA plus one poll of the others. False if it gave up.
__device__ bool grid_barrier(unsigned int* bar, const Smem& m) {
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned long long* ctr = reinterpret_cast<unsigned long long*>(bar);
        unsigned long long old;
        asm volatile("atom.add.acq_rel.gpu.u64 %0, [%1], 1;" : "=l"(old) : "l"(ctr) : "memory");
        const unsigned long long target = (old / gridDim.x + 1) * gridDim.x;
        bool ok = true;
        if (old + 1 != target) {
            const uint64_t t0 = global_timer_ns();
            while (true) {
                unsigned long long now;
                asm volatile("ld.acquire.gpu.u64 %0, [%1];" : "=l"(now) : "l"(ctr) : "memory");
                if (now >= target) break;
                if (global_timer_ns() - t0 > kWaitLimitNs) {
                    ok = false;
                    break;
                }
                __nanosleep(32);
            }
        }
        if (!ok) record_failure(m.info);
    }
    __syncthreads();
    return m.info[kInfoAbort] == 0;
}

template <int D, int BLK, int DG>
__global__ void __launch_bounds__(kStepThreads, 1)
    decode_step_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                       const Params p, const StepParams f) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const Smem m = setup_smem(smem_raw, p);
    if (threadIdx.x == 0) {
        prefetch_tensor_map(&tmK);
        prefetch_tensor_map(&tmV);
    }
    gate_phase<D, BLK, DG>(p, f, m);
    fence_proxy_async_smem();  // phase-1 use of the ring precedes phase-2 copies into it
    // One CTA per row in both phases: CTA r selects row r and then decodes it,
    // nothing crosses CTAs, and a CTA barrier is all phase 2 needs.
    if (f.gate_ctas == f.rows && p.P == f.rows) __syncthreads();
    else grid_barrier(f.grid_bar, m);
    if ((int)blockIdx.x >= p.P) return;  // more SMs than decode ranges
    const long long g0 = (long long)blockIdx.x * p.V / p.P;
    const long long g1 = (long long)(blockIdx.x + 1) * p.V / p.P;
    const int warp = threadIdx.x >> 5;
    if (warp == kConsumerWarps) decode_producer<D, BLK, true>(&tmK, &tmV, p, m, g0, g1);
    else if (warp >= kHelperWarp0) decode_helpers<D, BLK>(p, f, m, g0, g1);
    else decode_consumers<D, BLK, true>(p, f, m, g0, g1);
}

// One CTA waits, with the given limit, on an mbarrier that nothing ever
// arrives at; the wait must give up and report it.
__device__ int g_wait_selftest_result = -1;

__global__ void wait_selftest_kernel(unsigned long long limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(smem_addr(&bar), 1);
        fence_mbar_init();
    }
    __syncthreads();
    const bool completed = mbar_wait(smem_addr(&bar), 0u, limit_ns);
    __syncthreads();
    if (threadIdx.x == 0) g_wait_selftest_result = completed ? 0 : 1;
}

// ---------------------------------------------------------------- host side

struct Layout {
    int nst, stage_bytes, merge_off, info_off, bar_off, refresh_off, total;
};

template <int D, int BLK>
Layout make_layout(int G, bool with_refresh) {
    using C = Cfg<D, BLK>;
    Layout l;
    l.stage_bytes = (2 * C::kTileBytes + G * D * 2 + 1023) / 1024 * 1024;
    const int merge_bytes = kConsumerWarps * G * D * 4 + 2 * kConsumerWarps * G * 4;
    const int bar_bytes = (2 * kMaxStages + 2 + kMaxGateStages) * 8;
    const int refresh_bytes = with_refresh ? (int)sizeof(PoolSmem<D>) + 16 : 0;
    const int tail = merge_bytes + kInfoWords * 4 + bar_bytes + refresh_bytes + 64;
    int nst = (kSmemLimit - 1024 - tail) / l.stage_bytes;
    l.nst = nst > kMaxStages ? kMaxStages : nst;
    l.merge_off = l.nst * l.stage_bytes;
    l.info_off = (l.merge_off + merge_bytes + 15) / 16 * 16;
    l.bar_off = (l.info_off + kInfoWords * 4 + 15) / 16 * 16;
    l.refresh_off = l.bar_off + bar_bytes;
    l.total = l.refresh_off + refresh_bytes + 1024;  // + slack for the 1024-byte alignment
    return l;
}

template <int D, int BLK>
Params make_params(const Shape& s, const DecodeLaunch& a, const Layout& l, int P) {
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
    p.P = P;
    p.nst = l.nst;
    p.stage_bytes = l.stage_bytes;
    p.merge_off = l.merge_off;
    p.info_off = l.info_off;
    p.bar_off = l.bar_off;
    p.scale_log2 = a.sm_scale * kLog2e;
    return p;
}

template <typename K>
cudaError_t allow_big_smem(K kernel) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit);
}

template <int D, int BLK>
cudaError_t launch_impl(const Shape& s, const DecodeLaunch& a, const CUtensorMap& tmK, const CUtensorMap& tmV,
                        int num_sms, cudaStream_t stream) {
    const Layout l = make_layout<D, BLK>(s.G, false);
    if (l.nst < 2) return cudaErrorInvalidConfiguration;
    static bool attr_done = false;  // once per template instance (benign race)
    if (!attr_done) {
        cudaError_t e = allow_big_smem(sparse_decode_kernel<D, BLK>);
        if (e != cudaSuccess) return e;
        attr_done = true;
    }
    const Params p = make_params<D, BLK>(s, a, l, sparse_decode_ctas(s, a.kmax, a.num_splits, num_sms));
    sparse_decode_kernel<D, BLK><<<p.P, kThreads, l.total, stream>>>(tmK, tmV, p);
    return cudaGetLastError();
}

// Decode CTAs of the fused step. With no more rows than SMs every row gets
// the same whole number c of CTAs, so each CTA range is one piece of one row
// (no row hand-over in the middle of a stream; c = 1 writes the output
// directly); otherwise one CTA per SM over the positions laid end to end.
int step_decode_ctas(const Shape& s, int kmax, int num_sms) {
    const long long rows = (long long)s.B * s.Hkv;
    const long long V = rows * kmax;
    if (rows <= num_sms) {
        long long c = num_sms / rows;
        if (c > kmax) c = kmax;
        return (int)(rows * c);
    }
    return (int)(num_sms < V ? num_sms : V);
}

int step_num_splits(const Shape& s, int kmax, int num_sms) {
    const long long P = step_decode_ctas(s, kmax, num_sms);
    return (int)(kmax < P ? kmax : P);
}

template <int D, int BLK, int DG>
cudaError_t step_impl(const Shape& s, const StepLaunch& a, const CUtensorMap& tmK, const CUtensorMap& tmV,
                      int num_sms, cudaStream_t stream) {
    const Layout l = make_layout<D, BLK>(s.G, true);
    if (l.nst < 2) return cudaErrorInvalidConfiguration;
    const int keys_bytes = (s.NBmax * 4 + 1023) / 1024 * 1024;
    const int ring = l.nst * l.stage_bytes;
    const int n_gate = (ring - kGateScratchBytes - keys_bytes) / kGateChunkBytes;
    if (n_gate < 1) return cudaErrorInvalidConfiguration;
    static bool attr_done = false;
    if (!attr_done) {
        cudaError_t e = allow_big_smem(decode_step_kernel<D, BLK, DG>);
        if (e != cudaSuccess) return e;
        attr_done = true;
    }
    const int kmax = a.budget_tokens / s.blk;
    const long long V = (long long)s.B * s.Hkv * kmax;
    const int P = step_decode_ctas(s, kmax, num_sms);
    const int S = step_num_splits(s, kmax, num_sms);
    unsigned char* ws = static_cast<unsigned char*>(a.workspace);
    WorkspaceLayout wl = step_workspace_layout(s, kmax, num_sms);

    DecodeLaunch d;
    d.q = a.q;
    d.seq_lens = a.seq_lens;
    d.block_idx = a.block_idx;
    d.num_selected = a.num_selected;
    d.o_part = reinterpret_cast<float*>(ws + wl.o_part);
    d.lse_part = reinterpret_cast<float*>(ws + wl.lse_part);
    d.kmax = kmax;
    d.num_splits = S;
    d.sm_scale = a.sm_scale;
    const Params p = make_params<D, BLK>(s, d, l, P);

    StepParams f;
    f.k_cache = static_cast<const __nv_bfloat16*>(a.k_cache);
    f.w_q = a.w_q;
    f.w_k = a.w_k;
    f.upd_start = a.upd_start;
    f.kpool = a.kpool;
    f.block_idx = a.block_idx;
    f.num_selected = a.num_selected;
    f.out = static_cast<__nv_bfloat16*>(a.out);
    f.lse_out = a.lse_out;
    f.grid_bar = reinterpret_cast<unsigned int*>(ws + wl.grid_bar);
    f.row_done = reinterpret_cast<unsigned int*>(ws + wl.row_done);
    f.row_cnt = reinterpret_cast<unsigned int*>(ws + wl.row_cnt);
    f.qg_flag = reinterpret_cast<unsigned int*>(ws + wl.qg_flag);
    f.qg_g = reinterpret_cast<float*>(ws + wl.qg);
    f.keys_g = reinterpret_cast<uint32_t*>(ws + wl.keys);
    f.rows = s.B * s.Hkv;
    f.gate_ctas = f.rows <= num_sms ? f.rows * (num_sms / f.rows) : num_sms;
    f.NBmax = s.NBmax;
    f.dg = s.dg;
    f.refresh_off = l.refresh_off;
    f.keys_off = kGateScratchBytes;
    f.chunk_off = kGateScratchBytes + keys_bytes;
    f.n_gate_stages = n_gate > kMaxGateStages ? kMaxGateStages : n_gate;

    cudaLaunchConfig_t cfg = {};
    // With one CTA per row in both phases nothing crosses CTAs: a plain launch of
    // one CTA per row. Otherwise every SM, co-resident for the grid barrier.
    const bool barrier = !(f.gate_ctas == f.rows && P == f.rows);
    cfg.gridDim = dim3(barrier ? num_sms : f.rows, 1, 1);
    cfg.blockDim = dim3(kStepThreads, 1, 1);
    cfg.dynamicSmemBytes = l.total;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = barrier ? 1 : 0;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, decode_step_kernel<D, BLK, DG>, tmK, tmV, p, f);
    if (e != cudaSuccess) (void)cudaGetLastError();  // a rejected launch must not leak into the next call
    return e;
}

}  // namespace

WorkspaceLayout step_workspace_layout(const Shape& s, int kmax, int num_sms) {
    WorkspaceLayout w;
    const size_t rows = (size_t)s.B * s.Hkv;
    const size_t S = (size_t)step_num_splits(s, kmax, num_sms);
    auto up = [](size_t x) { return (x + 255) / 256 * 256; };
    w.grid_bar = 0;
    w.row_done = 256;
    w.row_cnt = up(w.row_done + rows * 4);
    w.qg_flag = up(w.row_cnt + rows * 4);
    w.counters_end = up(w.qg_flag + rows * 4);  // everything before this must start at zero
    w.qg = w.counters_end;
    w.keys = up(w.qg + rows * (size_t)s.dg * 4);
    w.o_part = up(w.keys + rows * (size_t)s.NBmax * 4);
    w.lse_part = up(w.o_part + (size_t)s.B * s.Hq * S * s.D * 4);
    w.total = up(w.lse_part + (size_t)s.B * s.Hq * S * 4);
    return w;
}

cudaError_t read_decode_wait_failures(unsigned int* count, bool reset) {
    cudaError_t e = cudaMemcpyFromSymbol(count, g_decode_wait_failures, sizeof(unsigned int));
    if (e != cudaSuccess || !reset) return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_decode_wait_failures, &zero, sizeof(unsigned int));
}

cudaError_t run_wait_selftest(unsigned long long limit_ns, int* timed_out) {
    const int unset = -1;
    cudaError_t e = cudaMemcpyToSymbol(g_wait_selftest_result, &unset, sizeof(int));
    if (e != cudaSuccess) return e;
    wait_selftest_kernel<<<1, 32>>>(limit_ns);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = cudaDeviceSynchronize()) != cudaSuccess) return e;
    int r = -1;
    if ((e = cudaMemcpyFromSymbol(&r, g_wait_selftest_result, sizeof(int))) != cudaSuccess) return e;
    *timed_out = r;
    return cudaSuccess;
}

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

// ---------------------------------------------------------------- step without a caller workspace
//
// Some callers cannot allocate device memory for the step's scratch: a plugin
// that its host framework hands nothing but input and output tensors, or a
// decode loop that must not call cudaMalloc (it can synchronise the device)
// once serving has started. For them the step's scratch lives in this
// file-scope array, one copy on every GPU that loads the library, held until
// the process exits. Its address is looked up once per device.
constexpr size_t kStaticScratchBytes = size_t(32) << 20;
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

size_t static_scratch_bytes() { return kStaticScratchBytes; }

cudaError_t launch_decode_step_static(const Shape& s, StepLaunch a, const CUtensorMap& tmK, const CUtensorMap& tmV,
                                      int num_sms, cudaStream_t stream) {
    constexpr int kMaxDevices = 64;
    static void* scratch[kMaxDevices] = {nullptr};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    if (!scratch[dev]) {  // set-up, once per device, with that device current
        void* ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_static_scratch);
        if (e != cudaSuccess) return e;
        scratch[dev] = ptr;
    }
    const WorkspaceLayout wl = step_workspace_layout(s, a.budget_tokens / s.blk, num_sms);
    if (wl.total > kStaticScratchBytes) return cudaErrorInvalidValue;
    // The array keeps the previous call's contents: the barrier words and row
    // counts must start at zero.
    e = cudaMemsetAsync(scratch[dev], 0, wl.counters_end, stream);
    if (e != cudaSuccess) return e;
    a.workspace = scratch[dev];
    return launch_decode_step(s, a, tmK, tmV, num_sms, stream);
}

cudaError_t launch_decode_step(const Shape& s, const StepLaunch& a, const CUtensorMap& tmK, const CUtensorMap& tmV,
                               int num_sms, cudaStream_t stream) {
#define SEER_STEP(D_, B_, G_) \
    if (s.D == D_ && s.blk == B_ && s.dg == G_) return step_impl<D_, B_, G_>(s, a, tmK, tmV, num_sms, stream)
    SEER_STEP(128, 64, 128);
    SEER_STEP(128, 128, 128);
    SEER_STEP(128, 64, 64);
    SEER_STEP(128, 128, 64);
    SEER_STEP(64, 64, 128);
    SEER_STEP(64, 128, 128);
    SEER_STEP(64, 64, 64);
    SEER_STEP(64, 128, 64);
#undef SEER_STEP
    return cudaErrorInvalidValue;
}

}  // namespace seer
