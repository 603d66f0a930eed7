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
//  * one producer warp: a single lane issues 2-D TMA tile loads (128-byte
//    swizzle) of the whole K and V tile of each kept block straight into a
//    ring of shared-memory stages, with an mbarrier pair per stage; the
//    decode query of a row rides along as a bulk copy with the first block
//    the CTA takes of that row. Loads carry an L2 evict-first hint (each
//    tile is read once).
//  * eight consumer warps, each owning a fixed slice of blk/8 tokens of every
//    block. Q K^T and P V run on the tensor cores (mma.sync bf16 -> fp32):
//    the G <= 8 query heads of the group form the M side (padded to 16),
//    tokens and head_dim the N / K sides, operands fetched with ldmatrix
//    (swizzle-matched, conflict-free). Each warp keeps its own online
//    softmax state; the eight states are merged through shared memory when
//    the CTA leaves a row.
//  * tokens t >= L_b of the partial last block are masked to -inf and their
//    V rows zeroed in shared memory before P V (the cache past L_b may hold
//    anything, NaN included).
//  * every wait is bounded (mbarrier waits and waits on other CTAs alike); on
//    expiry the CTA counts a failure, marks what it was producing with NaN
//    and leaves only after its own copies have landed.
//
// sparse_decode_kernel (seer_sparse_decode) splits the kept positions of all
// rows, laid end to end, into equal contiguous ranges, one per CTA, and writes
// one partial (o, lse) "slot" per (CTA, row) overlap; seer_combine merges them.
//
// decode_step_kernel (seer_decode_step) runs the whole step in one
// cooperative launch of one CTA per SM, with no grid-wide barrier:
//   gate: the pooled-key positions of all rows are split over the CTAs; each
//     projects the group's mean query of the rows it touches, scores their
//     cached pooled keys (streamed into the idle stage ring by bulk copies)
//     and the CTA that finishes a row selects its kept blocks -- with the
//     same arithmetic as the separate kernels (gate_core.cuh), so both paths
//     give bit-identical block lists -- then publishes the row (a release
//     flag tagged with the launch's epoch);
//   decode: every CTA then takes chunks of kept positions from rows that are
//     published, its own rows first, then any row with positions left (one
//     atomic claim per chunk), so all SMs stream until the last chunk and the
//     slower ones are relieved by the faster ones. A CTA keeps one online-
//     softmax state for as long as it stays on a row; when it leaves the row
//     it writes the row's output directly (it took every position) or a
//     partial slot, and the CTA that completes a row's positions merges its
//     slots into the output.
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
constexpr int kGateScratchBytes = 16384;  // gate scratch, in the merge area
constexpr int kGateChunkBytes = 32768;    // phase-1 bulk copy unit (pooled-K rows)
constexpr int kMinGatePositions = 32;     // fewest pooled-key rows worth a CTA of its own in the gate
constexpr int kMaxSmemDevices = 64;       // devices whose kernel attributes are tracked
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
    long long V;  // rows * kmax virtual positions (standalone decode)
    int Hq, Hkv, G, Lmax, kmax, S, P, nst;
    int stage_bytes, merge_off, info_off, bar_off;
    float scale_log2;  // sm_scale * log2(e)
};

// Shared-memory info words after the per-stage `valid` counts.
constexpr int kInfoAbort = kMaxStages;         // a wait of this CTA gave up
constexpr int kInfoMergeRow = kMaxStages + 1;  // this CTA merges the current row
constexpr int kInfoEpoch = kMaxStages + 2;     // launch epoch (fused step)
constexpr int kInfoWords = kMaxStages + 4;
// Fused step: what the producer tells the consumers about each stage.
constexpr int kStageInfoWords = 8;  // valid, row, flags, slot, positions of the run, positions of the row
constexpr int kRunStart = 1;        // first block of a run: reset the state, the row's query rides along
constexpr int kRunEnd = 2;          // last block of a run: write the run's result
constexpr int kRunWhole = 4;        // the run holds every position of its row: write the output directly
constexpr int kExit = 8;            // no more work: the consumers leave

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

// Shared-memory views common to both kernels. In the fused step, the gate's
// scratch (GateScratch) lives in the merge area, which the decode uses only
// later, so the whole stage ring can stream pooled keys.
struct Smem {
    unsigned char* base;  // 1024-aligned
    uint32_t sbase;
    float* merge;
    int* info;
    int* sinfo;  // [kMaxStages][kStageInfoWords] (fused step)
    uint32_t bars;
    int nst;
    __device__ __forceinline__ uint32_t full(int st) const { return bars + 8u * st; }
    __device__ __forceinline__ uint32_t empty(int st) const { return bars + 8u * (nst + st); }
    __device__ __forceinline__ uint32_t cons() const { return bars + 16u * nst; }
    __device__ __forceinline__ uint32_t gate(int st) const { return bars + 16u * nst + 8u + 8u * st; }
    __device__ __forceinline__ uint32_t helper() const { return bars + 16u * nst + 8u + 8u * kMaxGateStages; }
    __device__ __forceinline__ uint32_t wq() const { return bars + 16u * nst + 16u + 8u * kMaxGateStages; }
    __device__ __forceinline__ uint32_t thr() const { return bars + 16u * nst + 24u + 8u * kMaxGateStages; }
};

__device__ __forceinline__ Smem setup_smem(unsigned char* raw, const Params& p) {
    Smem m;
    m.base = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
    m.sbase = smem_addr(m.base);
    m.merge = reinterpret_cast<float*>(m.base + p.merge_off);
    m.info = reinterpret_cast<int*>(m.base + p.info_off);
    m.sinfo = m.info + kInfoWords;
    m.bars = m.sbase + p.bar_off;
    m.nst = p.nst;
    if (threadIdx.x == 0) {
        for (int st = 0; st < p.nst; ++st) {
            mbar_init(m.full(st), 1);
            mbar_init(m.empty(st), kConsumerWarps);
        }
        mbar_init(m.cons(), kConsumerWarps);  // one arrival per warp (warp_group_sync)
        for (int st = 0; st < kMaxGateStages; ++st) mbar_init(m.gate(st), 1);
        mbar_init(m.helper(), kHelperThreads / 32);
        mbar_init(m.wq(), 1);
        mbar_init(m.thr(), 1);
        for (int i = 0; i < kInfoWords; ++i) m.info[i] = 0;
        fence_mbar_init();
    }
    __syncthreads();
    return m;
}

// A group of whole warps meets on `bar` (initialised with the group's warp
// count): each warp reconverges, one lane arrives for it, every lane waits
// (bounded) and the warp reconverges again, so a warp whose lanes took
// different branches before the call (a lane subset doing extra work) can
// neither arrive in part nor leave in part. False if the wait gave up.
__device__ __forceinline__ bool warp_group_sync(uint32_t bar, uint32_t& phase, int* info) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
    const bool ok = mbar_wait(bar, phase);
    __syncwarp();
    phase ^= 1u;
    if (!ok) record_failure(info);
    return ok;
}

// All 8 consumer warps meet (bounded); false if the wait gave up.
__device__ __forceinline__ bool consumer_sync(const Smem& m, uint32_t& cph) {
    return warp_group_sync(m.cons(), cph, m.info);
}

// ---------------------------------------------------------------- one consumer warp's attention state

// The online-softmax state of one consumer warp over the tokens of its slice:
// row g of the mma fragments is query head g of the group (rows >= G idle).
template <int D, int BLK>
struct WarpState {
    float m_run, l_run;                          // running max (log2 domain) and sum of row g
    float o[Cfg<D, BLK>::kDTiles][4];            // unnormalised output, head_dim in n8 tiles
    uint32_t qa[Cfg<D, BLK>::kKSteps][2];        // A fragments of the group's queries
};

template <int D, int BLK>
__device__ __forceinline__ void ws_reset(WarpState<D, BLK>& w) {
    w.m_run = -INFINITY;
    w.l_run = 0.f;
#pragma unroll
    for (int dt = 0; dt < Cfg<D, BLK>::kDTiles; ++dt) w.o[dt][0] = w.o[dt][1] = w.o[dt][2] = w.o[dt][3] = 0.f;
}

// Query fragments from the bf16 [G, D] rows at qs (shared memory).
template <int D, int BLK>
__device__ __forceinline__ void ws_load_q(WarpState<D, BLK>& w, const __nv_bfloat16* qs, int G) {
    const int lane = threadIdx.x & 31, g = lane >> 2, tig = lane & 3;
#pragma unroll
    for (int kk = 0; kk < Cfg<D, BLK>::kKSteps; ++kk) {
        w.qa[kk][0] = g < G ? *reinterpret_cast<const uint32_t*>(qs + g * D + kk * 16 + 2 * tig) : 0u;
        w.qa[kk][1] = g < G ? *reinterpret_cast<const uint32_t*>(qs + g * D + kk * 16 + 8 + 2 * tig) : 0u;
    }
}

// Fold the warp's token slice [tbase, tbase + blk/8) of one staged K/V block
// (valid tokens < `valid`, valid > tbase) into the state. Returns true when it
// zeroed V rows in shared memory (the caller fences them before releasing the
// stage).
template <int D, int BLK>
__device__ __forceinline__ bool ws_block(WarpState<D, BLK>& w, uint32_t stK, int valid, int tbase, int G,
                                         float scale_log2) {
    using C = Cfg<D, BLK>;
    const int lane = threadIdx.x & 31, g = lane >> 2, tig = lane & 3;
    const uint32_t stV = stK + C::kTileBytes;
    bool wrote = false;
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
            mma_bf16_16816(sacc[0], w.qa[2 * kk2][0], 0u, w.qa[2 * kk2][1], 0u, r0, r1);
            mma_bf16_16816(s2, w.qa[2 * kk2 + 1][0], 0u, w.qa[2 * kk2 + 1][1], 0u, r2, r3);
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
            mma_bf16_16816(sacc[0], w.qa[kk][0], 0u, w.qa[kk][1], 0u, r0, r1);
            mma_bf16_16816(sacc[1], w.qa[kk][0], 0u, w.qa[kk][1], 0u, r2, r3);
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
            x[nt][e] = (t < valid) ? sacc[nt][e] * scale_log2 : -INFINITY;
            mloc = fmaxf(mloc, x[nt][e]);
        }
    }
    mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, 1));
    mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, 2));
    const float m_new = fmaxf(w.m_run, mloc);
    const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
    const float alpha = exp2f(w.m_run - m_use);
    float pv[C::kNT8][2];
    float psum = 0.f;
#pragma unroll
    for (int nt = 0; nt < C::kNT8; ++nt) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            pv[nt][e] = (g < G) ? exp2f(x[nt][e] - m_use) : 0.f;
            psum += pv[nt][e];
        }
    }
    w.l_run = w.l_run * alpha + psum;
    w.m_run = m_new;
#pragma unroll
    for (int dt = 0; dt < C::kDTiles; ++dt) {
        w.o[dt][0] *= alpha;
        w.o[dt][1] *= alpha;
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
            for (int u = 0; u < 4; ++u) mma_bf16_1688(w.o[dq * 4 + u], a0, 0u, b[u]);
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
            mma_bf16_16816(w.o[2 * dp], a0, 0u, a2, 0u, b0, b1);
            mma_bf16_16816(w.o[2 * dp + 1], a0, 0u, a2, 0u, b2, b3);
        }
    }
    return wrote;
}

// The warp's state into the CTA merge area: mO [8][G][D], mM / mL [8][G].
template <int D, int BLK>
__device__ __forceinline__ void ws_to_smem(WarpState<D, BLK>& w, const Smem& m, int G) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, tig = lane & 3;
    float* mO = m.merge;
    float* mM = m.merge + kConsumerWarps * G * D;
    float* mL = mM + kConsumerWarps * G;
    float l = w.l_run;
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    if (g < G) {
        if (tig == 0) {
            mM[warp * G + g] = w.m_run;
            mL[warp * G + g] = l;
        }
        float* dst = mO + (size_t)(warp * G + g) * D + 2 * tig;
#pragma unroll
        for (int dt = 0; dt < Cfg<D, BLK>::kDTiles; ++dt)
            *reinterpret_cast<float2*>(dst + dt * 8) = make_float2(w.o[dt][0], w.o[dt][1]);
    }
}

// Merge of the eight warp states in the merge area for element idx = h*D + d
// of the group: the normalised output value and the head's lse (natural log).
// Returns false when no warp saw a valid token (the value is then 0, lse -inf).
template <int D>
__device__ __forceinline__ bool merged_value(const Smem& m, int G, int idx, float& value, float& lse) {
    const float* mO = m.merge;
    const float* mM = m.merge + kConsumerWarps * G * D;
    const float* mL = mM + kConsumerWarps * G;
    const int h = idx / D, d = idx - h * D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, mM[w * G + h]);
    if (M == -INFINITY) {
        value = 0.f;
        lse = -INFINITY;
        return false;
    }
    float wsum = 0.f, acc = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) {
        const float mw = mM[w * G + h];
        if (mw != -INFINITY) {
            const float e = exp2f(mw - M);
            wsum += e * mL[w * G + h];
            acc += e * mO[(size_t)(w * G + h) * D + d];
        }
    }
    value = acc / wsum;
    lse = (M + log2f(wsum)) * kLn2;
    return true;
}

// ================================================================ standalone decode (seer_sparse_decode)

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

template <int D, int BLK>
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

template <int D, int BLK>
__device__ void decode_consumers(const Params& p, const Smem& m, long long g0, long long g1) {
    using C = Cfg<D, BLK>;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ctid = threadIdx.x;             // 0 .. 255
    const int tbase = warp * C::kTokPerWarp;  // this warp's token slice of each block
    int st = 0;
    uint32_t ph = 0, cph = 0;
    bool ok = true;
    WarpState<D, BLK> w;

    for (int r = (int)(g0 / p.kmax); ok && (long long)r * p.kmax < g1; ++r) {
        const Segment s = make_segment(p, r, g0, g1);
        const size_t head0 = (size_t)s.b * p.Hq + (size_t)s.kvh * p.G;
        if (s.a1 > s.a0) {
            ws_reset(w);
            for (int i = s.a0; i < s.a1; ++i) {
                const bool landed = mbar_wait(m.full(st), ph);
                __syncwarp();  // the lanes leave the wait together (ldmatrix / mma.sync below)
                if (!landed) {
                    record_failure(m.info);
                    ok = false;
                    break;
                }
                const int valid = m.info[st];
                const uint32_t stK = m.sbase + (uint32_t)st * p.stage_bytes;
                if (i == s.a0)
                    ws_load_q(w, reinterpret_cast<const __nv_bfloat16*>(m.base + (size_t)st * p.stage_bytes +
                                                                        2 * C::kTileBytes),
                              p.G);
                const bool wrote = (valid > tbase) && ws_block(w, stK, valid, tbase, p.G, p.scale_log2);
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
            ws_to_smem(w, m, p.G);
            if (!(ok = consumer_sync(m, cph))) break;
            for (int idx = ctid; idx < p.G * D; idx += kConsumerThreads) {
                const int h = idx / D, d = idx - h * D;
                float v, lse;
                merged_value<D>(m, p.G, idx, v, lse);
                p.o_part[((head0 + h) * p.S + s.slot) * D + d] = v;
                if (d == 0) p.lse_part[(head0 + h) * p.S + s.slot] = lse;
            }
            // the merge area is reused by the next segment
            if (!(ok = consumer_sync(m, cph))) break;
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

template <int D, int BLK>
__global__ void __launch_bounds__(kThreads, 1)  // 9 warps are allocated registers as 12: <= 168 each
    sparse_decode_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                         const Params p) {
    after_prior_grid();
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const Smem m = setup_smem(smem_raw, p);
    const long long g0 = (long long)blockIdx.x * p.V / p.P;
    const long long g1 = (long long)(blockIdx.x + 1) * p.V / p.P;
    if ((threadIdx.x >> 5) == kConsumerWarps) decode_producer<D, BLK>(&tmK, &tmV, p, m, g0, g1);
    else decode_consumers<D, BLK>(p, m, g0, g1);
}

// ================================================================ fused step (seer_decode_step)

// Per-row state of the decode phase (workspace, 32 bytes per row). `ready`
// holds the epoch of the launch that published the row's block list; the
// other words are valid only once `ready` equals the current epoch (the
// selecting CTA sets them before its release), so nothing needs resetting
// between launches.
//
// The row's list positions not yet taken are [front, back), both in one
// 64-bit word so that one atomic add takes a piece from either end: CTAs
// working through the row take `chunk` positions from the front, CTAs that
// come to help take half of what is left from the back. An add that finds
// front >= back takes nothing; the one add that makes front >= back is the
// one that counts the row as fully taken.
struct RowState {
    unsigned int ready;       // epoch of the launch that published the block list
    unsigned int nslots;      // partial slots handed out (one per run that may need merging)
    unsigned long long span;  // front (low 32 bits) | back (high 32 bits, signed)
    unsigned int done;        // list positions whose partial has been written
    unsigned int pad[3];
};

__device__ __forceinline__ int span_front(unsigned long long v) { return (int)(uint32_t)v; }
__device__ __forceinline__ int span_back(unsigned long long v) { return (int)(uint32_t)(v >> 32); }

// Extra arguments of the fused step.
struct StepParams {
    const __nv_bfloat16* k_cache;
    const float* w_q;
    const float* w_k;
    const int32_t* upd_start;
    float* kpool;
    int32_t* block_idx;     // gate output, decode input
    int32_t* num_selected;  // idem
    __nv_bfloat16* out;
    float* lse_out;
    unsigned long long* launch_ctr;    // grows by gridDim.x per launch: the launch's epoch
    unsigned int* rows_taken;          // [2] rows whose every list position is taken, by launch parity
    unsigned int* row_cnt;             // [rows] finished gate pieces per row (reset by the selecting CTA)
    RowState* rs;                      // [rows]
    uint32_t* keys_g;                  // [rows, NBmax] order keys of the block scores
    int rows, NBmax, dg;
    int gate_ctas;                           // CTAs of the gate
    int gate_cpr;                            // CTAs per row when rows fit the grid, else 0
    int chunk;                               // list positions per claim from the front
    int keys_off, chunk_off, n_gate_stages;  // gate keys and pooled-key copies inside the stage ring
    int wq_stages;                           // rows fit the grid: the last gate stages first hold W_q
    int n_early;                             // one CTA per row: decode stages issued during the selection
    int sel_off;                             // rows this CTA selected (shared memory, kMaxSelRows)
    int refresh_off;                         // pool scratch of the helper warps (outside the ring)
};

// First block to refresh for sequence b (upd_start, by default the token just appended).
__device__ __forceinline__ int refresh_start_block(const StepParams& f, int b, int L, int NB, int blk) {
    int st0 = f.upd_start ? f.upd_start[b] : L - 1;
    st0 = st0 < 0 ? 0 : st0;
    return min(st0 / blk, NB);
}

__device__ __forceinline__ unsigned int ld_acquire_u32(const unsigned int* p) {
    unsigned int v;
    asm volatile("ld.acquire.gpu.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ unsigned int ld_relaxed_u32(const unsigned int* p) {
    unsigned int v;
    asm volatile("ld.relaxed.gpu.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release_u32(unsigned int* p, unsigned int v) {
    asm volatile("st.release.gpu.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// The tally of rows whose every list position is taken. A launch counts in
// the word of its epoch's parity, which the previous launch cleared, and
// clears the other word for the next launch (launches on one workspace run in
// stream order). Counting is a fire-and-forget add: no thread waits on it.
// The launch's epoch from the launch counter's old value. The empty asm keeps
// the division (and so the wait for the counter's atomic) at the point of use:
// the atomic is issued at kernel entry and returns while the gate's loads run.
__device__ __forceinline__ uint32_t epoch_of(unsigned long long old_ctr) {
    asm volatile("" : "+l"(old_ctr));
    return (uint32_t)(old_ctr / gridDim.x) + 1u;  // every launch adds gridDim.x
}

__device__ __forceinline__ void count_taken_row(unsigned int* tally, uint32_t epoch) {
    atomicAdd(tally + (epoch & 1u), 1u);
}

// ---------------------------------------------------------------- fused step: gate

// One row of the rows a CTA meets in its gate range.
struct GateRow {
    int gi;                    // gate index: the row's place in the gate's position order
    int r, b, kvh, L, NB, js;  // js: first block whose pooled key is refreshed
    int s0, s1;                // cached positions [s0, s1) this CTA scores
    int scored;                // the row's choice needs scores
    int refresh_now;           // this CTA refreshes the competing blocks [js, NB-1) here
};
constexpr int kMaxBatchRows = 8;

// The barrier of the selection's 352 threads (warps 0 .. 10) when the last
// warp issues the first decode stages meanwhile; no other code uses id 1.
struct SelectGroupSync {
    __device__ __forceinline__ void operator()() const { named_barrier_sync(1, kStepThreads - 32); }
};

// Rows a CTA selected, kept for its decode producer (outside the stage ring):
// the CTA keeps the first chunk of each of them, so it starts streaming with
// no global round trip.
constexpr int kMaxSelRows = 32;
struct SelList {
    int count;
    int publish;  // rows fit the grid: the row this CTA selected, released after the gate (else -1)
    int own_len;  // rows fit the grid: the length of the row this CTA gated
    int early_count;            // one CTA per row: stages the gate issued during the selection
    int early_ids[kMaxStages];  // their blocks (certainly kept), ascending
    int thr_valid;              // the selection's first threshold bin, for the warp that issues them
    int thr_bstar;
    SelectBins thr_bins;
    int row[kMaxSelRows];
    int nsel[kMaxSelRows];
    int len[kMaxSelRows];
    int head[kMaxSelRows][kSelectHead];  // the first list entries of each
};
static_assert(sizeof(SelectBins) == 20 && sizeof(SelList) == 4556, "the host-side replica of the layout");

// The gate's scratch (in the merge area). Once a batch is scored only rows and
// last_of are read again: the selection's scratch overlays what precedes them
// (the padding makes room for it where the query arrays are smaller).
template <int D, int DG>
constexpr int gate_work_bytes() {
    return 4 * (kMaxBatchRows * D + kMaxBatchRows * DG + DG) + (int)sizeof(PoolSmem<D>);
}
template <int D, int DG>
struct GateScratch {
    alignas(16) float qbar[kMaxBatchRows][D];
    alignas(16) float qg[kMaxBatchRows][DG];
    alignas(16) float kp_new[DG];
    PoolSmem<D> pool;
    unsigned char pad[(int)sizeof(SelectSmem<kStepThreads>) > gate_work_bytes<D, DG>()
                          ? (int)sizeof(SelectSmem<kStepThreads>) - gate_work_bytes<D, DG>() + 16
                          : 16];
    GateRow rows[kMaxBatchRows];
    int last_of[kMaxBatchRows];
};
static_assert(sizeof(GateScratch<128, 128>) <= kGateScratchBytes, "gate scratch");
static_assert(sizeof(GateScratch<64, 128>) <= kGateScratchBytes, "gate scratch");
static_assert(sizeof(GateScratch<64, 64>) <= kGateScratchBytes, "gate scratch");
using GateScratchSmallest = GateScratch<64, 64>;
static_assert(offsetof(GateScratchSmallest, rows) >= sizeof(SelectSmem<kStepThreads>),
              "the selection's scratch before the gate rows");

// The gate's row order. Rows fit the grid: row i. Rows outnumber the CTAs:
// head-major (i = kvh * B + b), so the few consecutive rows a CTA gates share
// one head's W_q, which then arrives by one bulk copy.
__device__ __forceinline__ int gate_row(const StepParams& f, int Hkv, int i) {
    if (f.gate_cpr > 0) return i;
    const int B = f.rows / Hkv;
    return (i % B) * Hkv + i / B;
}

// The gate. The R x NBmax pooled-key positions (row-major, the layout of
// kpool) are cut into gate_ctas equal contiguous ranges (with rows <= SMs,
// each row into the same whole number of ranges). Each CTA projects the
// group-mean query of every row its range touches, streams the cached pooled
// keys of its range into the stage ring (bulk copies), scores them (a lane
// quad per key row) and, when the row is shared, writes order keys to the
// workspace. A per-row count of finished ranges tells the last CTA of a row to
// select its blocks and publish the row. The open last block is never a
// candidate, so its pooled key is refreshed by the helper warps during the
// decode; only blocks that compete (a refresh point before the last block)
// are refreshed here. `old_ctr` (the launch counter before this CTA's add) is
// valid in thread 0.
template <int D, int BLK, int DG, bool kManyRows>
__device__ void gate_phase(const CUtensorMap* tmK, const CUtensorMap* tmV, const Params& p, const StepParams& f,
                           const Smem& m, unsigned long long old_ctr) {
    constexpr int kThreads = kStepThreads;
    constexpr int kWarps = kThreads / 32;
    constexpr int kChunkRows = kGateChunkBytes / (DG * 4);
    constexpr int kVecD = D / 32;
    using WVec = typename std::conditional<kVecD == 4, float4, float2>::type;
    GateScratch<D, DG>& sm = *reinterpret_cast<GateScratch<D, DG>*>(m.merge);
    uint32_t* keys = reinterpret_cast<uint32_t*>(m.base + f.keys_off);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = lane >> 2, qlane = lane & 3;
    const float inv_sqrt_dg = 1.0f / sqrtf((float)DG);
    const long long V1 = (long long)f.rows * f.NBmax;
    const int G1 = f.gate_ctas;
    if ((int)blockIdx.x >= G1) return;
    const long long h0 = (long long)blockIdx.x * V1 / G1;
    const long long h1 = (long long)(blockIdx.x + 1) * V1 / G1;
    const bool whole_rows = G1 == f.rows;  // one CTA per row: keys stay in shared memory
    // Gate indices i with i * NBmax < h1, from the one holding h0: exactly the
    // rows whose [first, last] covering-CTA interval contains this CTA (an empty
    // range strictly inside a row still counts for that row).
    const int r_stop = (int)((h1 + f.NBmax - 1) / f.NBmax);
    int chunk_it = 0;  // bulk copies consumed so far (the same count on every thread)
    // When the first batch's rows share one head (always with one row per CTA), W_q of
    // that head arrives by one bulk copy into the last wq_stages gate stages, so
    // no register loads sit in front of the lengths and the first pooled-key
    // copies; those stages join the ring once the projection has read them.
    const int wq_stages = f.wq_stages;
    const int n_first = f.n_gate_stages - wq_stages;  // gate stages free before the projection
    const float* wq_s = reinterpret_cast<const float*>(m.base + f.chunk_off + n_first * kGateChunkBytes);
    int wq_uses = 0;  // W_q copies waited on so far: the phase of its barrier
    auto order = [&](int i) { return kManyRows ? gate_row(f, p.Hkv, i) : i; };
    if constexpr (!kManyRows) {
        if (wq_stages > 0 && tid == 0) {
            const uint32_t bytes = (uint32_t)(DG * D * 4);
            mbar_arrive_expect_tx(m.wq(), bytes);
            bulk_load(m.sbase + (uint32_t)(f.chunk_off + n_first * kGateChunkBytes),
                      f.w_q + (size_t)((int)(h0 / f.NBmax) % p.Hkv) * DG * D, bytes, m.wq());
        }
    }

    for (int gi0 = (int)(h0 / f.NBmax); gi0 < r_stop;) {
        const int nb = min(kMaxBatchRows, r_stop - gi0);
        const int kvh0 = order(gi0) % p.Hkv;
        bool one_head = true;
        if constexpr (kManyRows)
            for (int k = 1; k < nb; ++k) one_head &= order(gi0 + k) % p.Hkv == kvh0;
        // (first batch only: a later one starts its copies at the ring position the last
        // batch left, which need not leave the W_q stages free)
        const bool wq_on = wq_stages > 0 && (!kManyRows || (one_head && chunk_it == 0));
        if (kManyRows && wq_on && tid == 0) {  // the first batch: its stages are untouched
            const uint32_t bytes = (uint32_t)(DG * D * 4);
            mbar_arrive_expect_tx(m.wq(), bytes);
            bulk_load(m.sbase + (uint32_t)(f.chunk_off + n_first * kGateChunkBytes),
                      f.w_q + (size_t)kvh0 * DG * D, bytes, m.wq());
        }
        // ---- (1) before anything else reaches DRAM: the projection weights of the
        //      batch rows (first kQBatch outputs per warp), their lengths and
        //      group-mean queries -- all independent loads, issued together.
        //      Every row of the batch overlaps a non-empty range, and each CTA
        //      projects the rows it scores itself (no hand-off between CTAs).
        constexpr int kQBatch = 16;
        const int total_q = (h1 > h0 ? nb : 0) * DG;  // outputs ordered by batch row, then e
        int len_raw = 0, upd_raw = -1;
        if (tid < nb) {
            const int b = order(gi0 + tid) / p.Hkv;
            len_raw = load_early(p.seq_lens + b);
            if (f.upd_start) upd_raw = load_early(f.upd_start + b);
        }
        WVec w[kQBatch];
        if (total_q > 0 && !wq_on) {
#pragma unroll
            for (int u = 0; u < kQBatch; ++u) {
                const int o = min(warp + u * kWarps, total_q - 1);
                const int k = o / DG, e = o % DG;
                const int kvh = order(gi0 + k) % p.Hkv;
                load_early(w[u], f.w_q + ((size_t)kvh * DG + e) * D + lane * kVecD);
            }
        }

        if (tid < nb) {
            GateRow& g = sm.rows[tid];
            g.gi = gi0 + tid;
            g.r = order(g.gi);
            g.b = g.r / p.Hkv;
            g.kvh = g.r - g.b * p.Hkv;
            g.L = clamp_len(len_raw, p.Lmax);
            g.NB = (g.L + BLK - 1) / BLK;
            const int st0 = max(f.upd_start ? upd_raw : g.L - 1, 0);  // as refresh_start_block
            g.js = g.NB > 0 ? min(st0 / BLK, g.NB) : g.NB;
            const long long rs = (long long)g.gi * f.NBmax;
            const int i0 = (int)(h0 > rs ? h0 - rs : 0);
            const int i1 = (int)((h1 - rs) < f.NBmax ? (h1 - rs) : f.NBmax);
            const int kb = p.kmax < g.NB ? p.kmax : g.NB;
            const int ncand = g.NB - 1;
            g.scored = kb - 1 > 0 && kb - 1 < ncand;
            const int lim = g.scored ? min(g.js, ncand) : 0;
            g.s0 = min(i0, lim);
            g.s1 = min(i1, lim);
            g.refresh_now = g.js < ncand && g.js >= i0 && g.js < i1;
            if (f.gate_cpr > 0) reinterpret_cast<SelList*>(m.base + f.sel_off)->own_len = g.L;  // nb == 1
        }
        auto nchunks_of = [&](int k) { return (sm.rows[k].s1 - sm.rows[k].s0 + kChunkRows - 1) / kChunkRows; };
        auto count_chunks = [&]() {
            int n = 0;
            for (int k = 0; k < nb; ++k) n += nchunks_of(k);
            return n;
        };
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
        // ---- (2) stream the cached pooled keys; meanwhile project the batch rows' queries.
        //      One row per CTA: thread 0 wrote the row itself and issues its first
        //      copies before the group-mean query.
        if (tid == 0 && wq_on && nb == 1) {  // the row thread 0 just wrote
            const int n0 = count_chunks();
            for (int i = 0; i < min(n_first, n0); ++i) issue(i);
        }
        if (total_q > 0) {
            // W_q by bulk copy: warp 0 stays free for the lengths and the copies
            const int q0 = wq_on ? 32 : 0;
            for (int idx = tid - q0; idx >= 0 && idx < nb * D; idx += kThreads - q0) {
                const int k = idx / D, d = idx - k * D;
                const int row = order(gi0 + k), b = row / p.Hkv, kvh = row - b * p.Hkv;
                sm.qbar[k][d] = group_query_mean_at(p.q + ((size_t)b * p.Hq + (size_t)kvh * p.G) * D, p.G, D, d);
            }
        }
        __syncthreads();
        const int total_chunks = count_chunks();
        if (tid == 0 && !(wq_on && nb == 1))
            for (int c = 0; c < min(wq_on ? n_first : f.n_gate_stages, total_chunks); ++c) issue(c);
        if (wq_on) {
            // the same pieces and sums as the register path below (equal bits); one
            // W_q row piece serves every row of the batch
            constexpr int kPerWarp = (DG + kWarps - 1) / kWarps;
            if (!mbar_wait(m.wq(), (uint32_t)(wq_uses & 1))) record_failure(m.info);
            ++wq_uses;
#pragma unroll 1
            for (int u0 = 0; u0 < kPerWarp; u0 += 4) {  // four W_q rows per warp in flight
                WVec wv[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int e = min(warp + (u0 + u) * kWarps, DG - 1);
                    wv[u] = *reinterpret_cast<const WVec*>(wq_s + (size_t)e * D + lane * kVecD);
                }
                if (!kManyRows || nb == 1) {
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int e = warp + (u0 + u) * kWarps;
                        const float x = warp_sum(piece_dot(wv[u], &sm.qbar[0][lane * kVecD]));
                        if (lane == 0 && e < DG) sm.qg[0][e] = x;
                    }
                } else {
#pragma unroll 1
                    for (int k = 0; k < nb; ++k)
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const int e = warp + (u0 + u) * kWarps;
                            const float x = warp_sum(piece_dot(wv[u], &sm.qbar[k][lane * kVecD]));
                            if (lane == 0 && e < DG) sm.qg[k][e] = x;
                        }
                }
            }
            fence_proxy_async_smem();  // these generic reads of W_q precede the copies into its stages
        } else if (total_q > 0) {
#pragma unroll
            for (int u = 0; u < kQBatch; ++u) {
                const int o = warp + u * kWarps;
                const int oc = min(o, total_q - 1);
                const int k = oc / DG, e = oc % DG;
                const float x = warp_sum(piece_dot(w[u], &sm.qbar[k][lane * kVecD]));
                if (lane == 0 && o < total_q) sm.qg[k][e] = x;
            }
            for (int o0 = warp + kQBatch * kWarps; o0 < total_q; o0 += 8 * kWarps) {  // batches beyond the first
                WVec w2[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int o = min(o0 + u * kWarps, total_q - 1);
                    const int k = o / DG, e = o % DG;
                    w2[u] = *reinterpret_cast<const WVec*>(f.w_q + ((size_t)sm.rows[k].kvh * DG + e) * D + lane * kVecD);
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int o = o0 + u * kWarps;
                    const int oc = min(o, total_q - 1);
                    const int k = oc / DG, e = oc % DG;
                    const float x = warp_sum(piece_dot(w2[u], &sm.qbar[k][lane * kVecD]));
                    if (lane == 0 && o < total_q) sm.qg[k][e] = x;
                }
            }
        }
        __syncthreads();
        if (tid == 0 && wq_on)  // the W_q stages are read: they join the ring
            for (int c = n_first; c < min(f.n_gate_stages, total_chunks); ++c) issue(c);

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
        //      the last CTA of a row selects its blocks and publishes the row
        __syncthreads();  // every key of the batch written before the adds
        if (tid < nb) {
            const GateRow& g = sm.rows[tid];
            const long long rs = (long long)g.gi * f.NBmax;
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
        SelectSmem<kThreads>& ssm = *reinterpret_cast<SelectSmem<kThreads>*>(m.merge);  // over the query arrays
        SelList& sel = *reinterpret_cast<SelList*>(m.base + f.sel_off);
        for (int k = 0; k < nb; ++k) {
            if (!sm.last_of[k]) continue;
            const GateRow& g = sm.rows[k];
            const int kb = p.kmax < g.NB ? p.kmax : g.NB;
            if (g.scored && !whole_rows)
                for (int i = tid; i < g.NB - 1; i += kThreads) keys[i] = __ldcg(f.keys_g + (size_t)g.r * f.NBmax + i);
            int kept = 0;  // thread 0: positions this CTA keeps
            const int si = sel.count;  // read by every thread before thread 0 may append
            __syncthreads();
            if (tid == 0) {
                f.num_selected[g.r] = kb;
                f.row_cnt[g.r] = 0u;  // ready for the next call: every CTA of the row has counted in
                // this CTA lists the row for its producer when it can, and, when rows
                // outnumber the CTAs (positions are then taken from the row's span),
                // keeps the row's first chunk
                const bool keep = kb > 0 && sel.count < kMaxSelRows;
                kept = (keep && f.gate_cpr == 0) ? min(f.chunk, kb) : 0;
                f.rs[g.r].span = ((unsigned long long)(uint32_t)kb << 32) | (uint32_t)kept;
                f.rs[g.r].nslots = 0u;
                f.rs[g.r].done = 0u;
                if (keep) {
                    sel.row[sel.count] = g.r;
                    sel.nsel[sel.count] = kb;
                    sel.len[sel.count] = g.L;
                    ++sel.count;
                }
            }
            __syncthreads();
            int32_t* list = f.block_idx + (size_t)g.r * p.kmax;
            int32_t* head = si < kMaxSelRows ? sel.head[si] : nullptr;
            if (whole_rows && f.n_early > 0 && kb > 0) {
                // One CTA per row: once the first histogram fixes the threshold bin, every
                // candidate above it is kept whatever the rest of the search finds. Warps
                // 0 .. 10 select (meeting at a named barrier); the last warp waits for that
                // bin and meanwhile starts the decode on the first such candidates.
                constexpr int kSelThreads = kThreads - 32;
                if (warp == kWarps - 1) {
                    const bool got = mbar_wait(m.thr(), 0u);
                    __syncwarp();
                    if (!got) record_failure(m.info);
                    int n = 0;
                    if (got && sel.thr_valid) {
                        using C = Cfg<D, BLK>;
                        constexpr unsigned kFull = 0xffffffffu;
                        const SelectBins bins = sel.thr_bins;
                        const int bstar = sel.thr_bstar;
                        const int ncand = g.NB - 1;
                        const uint64_t policy = l2_policy_evict_first();
                        const uint32_t qbytes = (uint32_t)(p.G * D * 2);
                        for (int i0 = 0; i0 < ncand && n < f.n_early; i0 += 32) {
                            const int i = i0 + lane;
                            unsigned msk = __ballot_sync(kFull, i < ncand && bins(keys[i]) > bstar);
                            while (msk != 0u && n < f.n_early) {
                                const int j = i0 + __ffs(msk) - 1;  // a full block: j < NB - 1
                                msk &= msk - 1u;
                                if (lane == 0) {  // stage n of a fresh ring: its empty phase has passed
                                    int* sinfo = m.sinfo + n * kStageInfoWords;
                                    sinfo[0] = BLK;
                                    sinfo[1] = g.r;
                                    sinfo[2] = n == 0 ? kRunStart : 0;
                                    sinfo[3] = 0;
                                    sinfo[4] = n + 1;
                                    sinfo[5] = kb;
                                    const uint32_t fb = m.full(n);
                                    mbar_arrive_expect_tx(fb, 2u * C::kTileBytes + (n == 0 ? qbytes : 0u));
                                    const uint32_t stK = m.sbase + (uint32_t)n * p.stage_bytes;
                                    const int y = g.r * p.Lmax + j * BLK;
#pragma unroll
                                    for (int bx = 0; bx < C::kBoxes; ++bx) {
                                        tma_load_2d(stK + bx * C::kBoxBytes, tmK, fb, bx * 64, y, policy);
                                        tma_load_2d(stK + C::kTileBytes + bx * C::kBoxBytes, tmV, fb, bx * 64, y,
                                                    policy);
                                    }
                                    if (n == 0)
                                        bulk_load(stK + 2 * C::kTileBytes,
                                                  p.q + ((size_t)g.b * p.Hq + (size_t)g.kvh * p.G) * D, qbytes, fb);
                                    sel.early_ids[n] = j;
                                }
                                ++n;
                            }
                        }
                    }
                    if (lane == 0) sel.early_count = n;
                } else {
                    auto threshold = [&](const SelectBins& bins, int bstar) {
                        if (tid == 0) {
                            sel.thr_bins = bins;
                            sel.thr_bstar = bstar;
                            sel.thr_valid = 1;
                            mbar_arrive(m.thr());  // releases these writes to the waiting warp
                        }
                    };
                    SelectSmem<kSelThreads>& ssm_g = *reinterpret_cast<SelectSmem<kSelThreads>*>(m.merge);
                    select_row<kSelThreads>(keys, g.NB, p.kmax, list, ssm_g, head, threshold, SelectGroupSync());
                    if (tid == 0 && !sel.thr_valid) mbar_arrive(m.thr());  // no threshold pass: nothing early
                }
            } else {
                select_row<kThreads>(keys, g.NB, p.kmax, list, ssm, head);
            }
            if (kb == 0) {  // a row without tokens is written here
                const size_t head0 = (size_t)g.b * p.Hq + (size_t)g.kvh * p.G;
                for (int i = tid; i < p.G * D; i += kThreads) f.out[head0 * D + i] = __float2bfloat16(0.f);
                if (tid < p.G && f.lse_out) f.lse_out[head0 + tid] = -INFINITY;
            }
            __syncthreads();  // the list, the count and the state before the release
            if (tid == 0) {
                if (f.gate_cpr > 0) {
                    sel.publish = g.r;  // released after the gate, so the producer starts first
                } else {
                    const uint32_t epoch = epoch_of(old_ctr);
                    if (kept == kb) count_taken_row(f.rows_taken, epoch);  // nothing left to take
                    st_release_u32(&f.rs[g.r].ready, epoch);
                }
            }
        }
        fence_proxy_async_smem();
        __syncthreads();  // scratch, keys and stages are reused by the next batch
        gi0 += nb;
    }
}

// ---------------------------------------------------------------- fused step: decode producer

// The producer warp of the decode phase. A run is the blocks a CTA takes of
// one row in one visit; the stage info tells the consumers where a run starts
// and ends. When rows fit the grid, the CTAs that gated a row (they all start
// once it is published) stream even, fixed parts of its list, and a row held
// by one CTA is written straight to the output. When rows outnumber the CTAs
// (rows then differ in length, and HBM serves SMs unevenly), the CTA streams
//   1. the rows it selected, from the first chunk it kept, then pieces from
//      the front (an atomic add on the row's span, issued one piece ahead of
//      its use) of an eighth of what is left, at least a chunk;
//   2. its other home rows, once published, from the front likewise;
//   3. then, while any row has at least two chunks left, half of what is left
//      of the row with the most left, from the back (one add), at most an
//      even share of all the rows' positions per CTA;
// and leaves once every row is fully taken.
template <int D, int BLK>
__device__ void step_producer(const CUtensorMap* tmK, const CUtensorMap* tmV, const Params& p, const StepParams& f,
                              const Smem& m) {
    using C = Cfg<D, BLK>;
    const int lane = threadIdx.x & 31;
    constexpr unsigned kFull = 0xffffffffu;
    const uint32_t epoch = (uint32_t)m.info[kInfoEpoch];
    const uint64_t policy = l2_policy_evict_first();
    const int R = f.rows;
    const int chunk = f.chunk;
    const uint32_t qbytes = (uint32_t)(p.G * D * 2);
    const SelList& sel = *reinterpret_cast<const SelList*>(m.base + f.sel_off);
    int st = 0;
    uint32_t ph = 0;
    long long issued = 0;
    bool ok = true;

    // One stage: block j (valid tokens `valid`, none when 0) of `row` with its flags.
    auto put = [&](int row, int j, int valid, int flags, int slot, int nrun, int nsel, bool with_q) {
        int good = 1;
        if (lane == 0) {
            if (!mbar_wait(m.empty(st), ph ^ 1u)) {
                good = 0;
                record_failure(m.info);
            } else {
                int* si = m.sinfo + st * kStageInfoWords;
                si[0] = valid;
                si[1] = row;
                si[2] = flags;
                si[3] = slot;
                si[4] = nrun;
                si[5] = nsel;
                const uint32_t fb = m.full(st);
                const uint32_t bytes = (valid > 0 ? 2u * C::kTileBytes : 0u) + (with_q ? qbytes : 0u);
                if (bytes) mbar_arrive_expect_tx(fb, bytes);
                else mbar_arrive(fb);
                const uint32_t stK = m.sbase + (uint32_t)st * p.stage_bytes;
                if (valid > 0) {
                    const int y = row * p.Lmax + j * BLK;
#pragma unroll
                    for (int bx = 0; bx < C::kBoxes; ++bx) {
                        tma_load_2d(stK + bx * C::kBoxBytes, tmK, fb, bx * 64, y, policy);
                        tma_load_2d(stK + C::kTileBytes + bx * C::kBoxBytes, tmV, fb, bx * 64, y, policy);
                    }
                }
                if (with_q) {
                    const int b = row / p.Hkv, kvh = row - b * p.Hkv;
                    bulk_load(stK + 2 * C::kTileBytes, p.q + ((size_t)b * p.Hq + (size_t)kvh * p.G) * D, qbytes, fb);
                }
                ++issued;
            }
        }
        ok = __shfl_sync(kFull, good, 0) != 0;
        if (ok && ++st == p.nst) {
            st = 0;
            ph ^= 1u;
        }
    };

    // A claim of `n` positions from the front (lane 0): its piece [a0, a1), empty
    // when a0 >= a1; the claim that takes the row's last position counts the row.
    auto take_front = [&](unsigned long long old, int n, int& a0, int& a1) {
        const int f0 = span_front(old), b0 = span_back(old);
        a0 = f0;
        a1 = min(f0 + n, b0);
        if (f0 < b0 && f0 + n >= b0) count_taken_row(f.rows_taken, epoch);
    };

    // Stream one run of `row` (nsel list positions) from the piece [a0, a1) it holds;
    // from the front, further pieces are claimed one ahead until the row has none left.
    // `ne` > 0: stages 0 .. ne-1 were issued by the gate (blocks sel.early_ids,
    // the run's start); those blocks are skipped here (never the list's last).
    auto run = [&](int row, int nsel, int a0, int a1, bool from_front, const int* head, int fixed_slot, int Lrow,
                   int ne) {
        const int b = row / p.Hkv;
        const int L = Lrow >= 0 ? Lrow : clamp_len(p.seq_lens[b], p.Lmax);
        const int NB = (L + BLK - 1) / BLK;
        const int32_t* list = f.block_idx + (size_t)row * p.kmax;
        unsigned int slot = 0;
        unsigned long long c1 = 0;  // lane 0: the claim in flight, of n1 positions
        int n1 = chunk;
        if (lane == 0) {
            slot = fixed_slot >= 0 ? (unsigned int)fixed_slot : atomicAdd(&f.rs[row].nslots, 1u);  // needed at the run's end
            if (from_front) {
                n1 = max(chunk, (nsel - a1) / 8);  // an eighth of what may be left, at least a chunk
                c1 = atomicAdd(&f.rs[row].span, (unsigned long long)n1);
            }
        }
        __syncwarp();
        int wbase = a0;  // the lanes hold list[wbase + lane]; a list this CTA selected starts in shared memory
        int jl = head ? head[lane] : ((a0 + lane < p.kmax) ? __ldcg(list + a0 + lane) : -1);
        const int early_id = lane < ne ? sel.early_ids[lane] : -1;
        int nrun = 0;
        bool first = ne == 0;
        while (ok) {
            const int cnt = a1 - a0;
            int na0 = 0, na1 = 0;
            for (int k = 0; ok && k < cnt; ++k) {
                const int pos = a0 + k;
                if (pos >= wbase + 32) {
                    wbase = pos;
                    jl = (pos + lane < p.kmax) ? __ldcg(list + pos + lane) : -1;
                }
                const int j = __shfl_sync(kFull, jl, pos - wbase);
                if (ne > 0 && k + 1 < cnt && __any_sync(kFull, early_id == j)) continue;
                const int valid = (j >= 0 && j < NB) ? min(BLK, L - j * BLK) : 0;
                int flags = first ? kRunStart : 0;
                if (k + 1 == cnt) {  // the run goes on with the claim in flight, if it took anything
                    int e0 = 0, e1 = 0;
                    if (lane == 0 && from_front) take_front(c1, n1, e0, e1);
                    na0 = __shfl_sync(kFull, e0, 0);
                    na1 = __shfl_sync(kFull, e1, 0);
                    if (na0 >= na1) {
                        flags |= kRunEnd;
                        if (nrun + cnt == nsel) flags |= kRunWhole;
                    } else if (na0 < wbase || na0 >= wbase + 32) {  // its indices travel during this stage's wait
                        wbase = na0;
                        jl = (na0 + lane < p.kmax) ? __ldcg(list + na0 + lane) : -1;
                    }
                }
                put(row, j, valid, flags, (int)slot, nrun + cnt, nsel, first);
                first = false;
            }
            nrun += cnt;
            if (na0 >= na1 || !ok) return;
            a0 = na0;
            a1 = na1;
            if (lane == 0) {
                n1 = max(chunk, (span_back(c1) - a1) / 8);
                c1 = atomicAdd(&f.rs[row].span, (unsigned long long)n1);
            }
        }
    };

    // Wait (bounded) until `row` is published; false if the wait gave up. The
    // acquire by lane 0, then the warp barrier, order the warp's reads of what
    // the selecting CTA wrote.
    auto wait_ready = [&](int row) {
        int good = 1;
        if (lane == 0 && ld_acquire_u32(&f.rs[row].ready) != epoch) {
            const uint64_t t0 = global_timer_ns();
            while (ld_acquire_u32(&f.rs[row].ready) != epoch) {
                if (global_timer_ns() - t0 > kWaitLimitNs) {
                    good = 0;
                    record_failure(m.info);
                    break;
                }
                __nanosleep(64);
            }
        }
        __syncwarp();
        return __shfl_sync(kFull, good, 0) != 0;
    };

    // A visit from the front of a published row this CTA did not select.
    auto visit_front = [&](int row) {
        int a0 = 0, a1 = 0, nsel = 0;
        if (lane == 0) {
            nsel = __ldcg(f.num_selected + row);
            take_front(atomicAdd(&f.rs[row].span, (unsigned long long)chunk), chunk, a0, a1);
        }
        a0 = __shfl_sync(kFull, a0, 0);
        a1 = __shfl_sync(kFull, a1, 0);
        nsel = __shfl_sync(kFull, nsel, 0);
        if (a0 < a1) run(row, nsel, a0, a1, true, nullptr, -1, -1, 0);
    };

    const int nselrows = sel.count;
    if (f.gate_cpr > 0) {
        // ---- rows fit the grid: the CTAs that gated a row (all start together
        //      once it is published) stream even, fixed parts of its list; a row
        //      held by one CTA is written straight to the output. The spare CTAs
        //      have no part.
        if ((int)blockIdx.x < f.gate_ctas) {
            const int row = (int)blockIdx.x / f.gate_cpr, part = (int)blockIdx.x % f.gate_cpr;
            int nsel = -1;
            const int* head = nullptr;
            for (int i = 0; i < nselrows; ++i)
                if (sel.row[i] == row) {
                    nsel = sel.nsel[i];
                    head = sel.head[i];
                }
            if (nsel < 0 && (ok = wait_ready(row))) {
                int v = 0;
                if (lane == 0) v = __ldcg(f.num_selected + row);
                nsel = __shfl_sync(kFull, v, 0);
            }
            if (ok) {
                const int a0 = (int)((long long)part * nsel / f.gate_cpr);
                const int a1 = (int)((long long)(part + 1) * nsel / f.gate_cpr);
                // a fixed slot per non-empty part: the merge adds the parts in the same
                // order on every call, so the output is the same bit for bit
                const int slot = nsel >= f.gate_cpr ? part : a0;
                // one CTA per row: the gate may have issued the first stages already
                const int ne = f.gate_cpr == 1 ? sel.early_count : 0;
                st = ne;  // < nst: the ring has not wrapped
                issued = ne;
                if (a0 < a1) run(row, nsel, a0, a1, false, a0 == 0 ? head : nullptr, slot, sel.own_len, ne);
            }
        }
        if (ok) put(0, 0, 0, kExit, 0, 0, 0, false);
        if (lane == 0)
            for (long long it = (issued > p.nst ? issued - p.nst : 0); it < issued; ++it) {
                const int s_it = (int)(it % p.nst);
                const uint32_t par = (uint32_t)((it / p.nst) & 1);
                if (!ok || !mbar_wait(m.empty(s_it), par)) (void)mbar_wait(m.full(s_it), par);
            }
        return;
    }

    // ---- rows outnumber the CTAs:
    // ---- 1. the rows this CTA selected, from the chunk it kept
    for (int i = 0; ok && i < nselrows; ++i)
        run(sel.row[i], sel.nsel[i], 0, min(chunk, sel.nsel[i]), true, sel.head[i], -1, sel.len[i], 0);

    // ---- 2. its other home rows
    int home_lo, home_hi;
    home_lo = (int)((long long)blockIdx.x * R / gridDim.x);
    home_hi = (int)((long long)(blockIdx.x + 1) * R / gridDim.x);
    for (int hr = home_lo; ok && hr < home_hi; ++hr) {
        const int row = gate_row(f, p.Hkv, hr);
        bool mine = false;
        for (int i = 0; i < nselrows; ++i) mine |= sel.row[i] == row;
        if (mine) continue;
        if (!(ok = wait_ready(row))) break;
        visit_front(row);
    }

    // ---- 3. help: half of what is left of the row with the most left (at most one CTA's
    //      even share of all rows' positions), from the back
    const int fair = (int)(((long long)R * p.kmax + gridDim.x - 1) / gridDim.x);
    int pos = home_hi % R;
    const int nwin = R < 32 ? R : 32;
    int empty_windows = 0;
    uint64_t idle_since = 0;
    while (ok) {
        unsigned int tally = 0;
        if (lane == 0) tally = ld_relaxed_u32(f.rows_taken + (epoch & 1u));
        int r = pos + lane;
        if (r >= R) r -= R;
        int left = -1;  // positions left; -1 not published yet
        if (lane < nwin && ld_relaxed_u32(&f.rs[r].ready) == epoch) {
            const unsigned long long sp = ld_relaxed_u64(&f.rs[r].span);
            left = max(0, span_back(sp) - span_front(sp));
        }
        int best = left, best_lane = lane;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {  // most left, lowest lane on ties
            const int ob = __shfl_xor_sync(kFull, best, o), ol = __shfl_xor_sync(kFull, best_lane, o);
            if (ob > best || (ob == best && ol < best_lane)) {
                best = ob;
                best_lane = ol;
            }
        }
        if (best >= 2 * chunk) {
            const int row = __shfl_sync(kFull, r, best_lane);
            int a0 = 0, a1 = 0, nsel = 0;
            if (lane == 0) {
                (void)ld_acquire_u32(&f.rs[row].ready);  // orders this warp's reads of the row's list
                nsel = __ldcg(f.num_selected + row);
                const int t = max(chunk, min(best / 2, fair));
                const unsigned long long old =
                    atomicAdd(&f.rs[row].span, (unsigned long long)0 - ((unsigned long long)(uint32_t)t << 32));
                const int f0 = span_front(old), b0 = span_back(old);
                a0 = max(b0 - t, f0);
                a1 = b0;
                if (f0 < b0 && b0 - t <= f0) count_taken_row(f.rows_taken, epoch);
            }
            __syncwarp();
            a0 = __shfl_sync(kFull, a0, 0);
            a1 = __shfl_sync(kFull, a1, 0);
            nsel = __shfl_sync(kFull, nsel, 0);
            if (a0 < a1) run(row, nsel, a0, a1, false, nullptr, -1, -1, 0);
            empty_windows = 0;
            idle_since = 0;
            continue;  // look at the same window again
        }
        int done = 0;
        if (lane == 0) done = tally >= (unsigned int)R;
        if (__shfl_sync(kFull, done, 0)) break;
        pos += nwin;
        if (pos >= R) pos -= R;
        if (++empty_windows * nwin >= R) {  // a whole pass found nothing to take: back off, bounded
            empty_windows = 0;
            if (lane == 0) {
                const uint64_t now = global_timer_ns();
                if (idle_since == 0) idle_since = now;
                else if (now - idle_since > kWaitLimitNs) {
                    record_failure(m.info);
                    ok = false;
                }
                __nanosleep(256);
            }
            ok = __shfl_sync(kFull, (int)ok, 0) != 0;
        }
    }
    if (ok) put(0, 0, 0, kExit, 0, 0, 0, false);  // the consumers leave after this stage
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

// ---------------------------------------------------------------- fused step: decode consumers

// The end of a run: the eight warp states are merged; a run that held every
// position of its row writes the output directly, any other run writes its
// slot and counts its positions, and the CTA whose count completes the row
// merges the row's slots (log-sum-exp weights) into the output.
template <int D, int BLK>
__device__ __forceinline__ bool step_flush(const Params& p, const StepParams& f, const Smem& m,
                                           WarpState<D, BLK>& w, const int* si, uint32_t& cph) {
    const int row = si[1], flags = si[2], slot = si[3], nrun = si[4], nsel = si[5];
    const int ctid = threadIdx.x;
    const int b = row / p.Hkv, kvh = row - b * p.Hkv;
    const size_t head0 = (size_t)b * p.Hq + (size_t)kvh * p.G;
    const bool whole = (flags & kRunWhole) != 0;
    ws_to_smem(w, m, p.G);
    if (!consumer_sync(m, cph)) return false;
    if (!whole && slot >= p.S) {  // cannot happen: runs per row <= slots (see step_geometry)
        if (ctid == 0) record_failure(m.info);
        return false;
    }
    for (int idx = ctid; idx < p.G * D; idx += kConsumerThreads) {
        const int h = idx / D, d = idx - h * D;
        float v, lse;
        merged_value<D>(m, p.G, idx, v, lse);
        if (whole) {
            f.out[(head0 + h) * D + d] = __float2bfloat16(v);
            if (d == 0 && f.lse_out) f.lse_out[head0 + h] = lse;
        } else {
            p.o_part[((head0 + h) * p.S + slot) * D + d] = v;
            if (d == 0) p.lse_part[(head0 + h) * p.S + slot] = lse;
        }
    }
    if (!consumer_sync(m, cph)) return false;  // the slot's writes before the count; the merge area is free
    if (whole) return true;
    if (ctid == 0) {
        const unsigned int before = atomic_add_acq_rel(&f.rs[row].done, (unsigned int)nrun);
        // every run of the row took its slot before it counted: the last count sees them all;
        // fixed parts (rows fit the grid) fill slots 0 .. min(nsel, parts) - 1
        const int ns = (before + (unsigned int)nrun != (unsigned int)nsel) ? 0
                       : f.gate_cpr > 0                                    ? min(nsel, f.gate_cpr)
                                                                           : (int)ld_relaxed_u32(&f.rs[row].nslots);
        *reinterpret_cast<volatile int*>(m.info + kInfoMergeRow) = min(ns, p.S);
    }
    __syncwarp();
    if (!consumer_sync(m, cph)) return false;  // the acquire, then every consumer reads the slots
    const int ns = *reinterpret_cast<volatile int*>(m.info + kInfoMergeRow);
    if (ns == 0) return true;
    float* wt = m.merge;  // [G][ns]: the slots' lse, then their normalised weights
    for (int i = ctid; i < p.G * ns; i += kConsumerThreads) {
        const int h = i / ns;
        wt[i] = __ldcg(p.lse_part + (head0 + h) * p.S + (i - h * ns));
    }
    if (!consumer_sync(m, cph)) return false;
    if (ctid < p.G) {
        float* l = wt + ctid * ns;
        float M = -INFINITY;
        for (int k = 0; k < ns; ++k) M = fmaxf(M, l[k]);
        float wsum = 0.f;
        for (int k = 0; k < ns; ++k) {
            const float e = (l[k] == -INFINITY || M == -INFINITY) ? 0.f : expf(l[k] - M);
            l[k] = e;
            wsum += e;
        }
        const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
        for (int k = 0; k < ns; ++k) l[k] *= inv;
        if (f.lse_out) f.lse_out[head0 + ctid] = (M == -INFINITY) ? -INFINITY : M + logf(wsum);
    }
    __syncwarp();
    if (!consumer_sync(m, cph)) return false;
    for (int idx = ctid; idx < p.G * D; idx += kConsumerThreads) {
        const int h = idx / D, d = idx - h * D;
        const float* src = p.o_part + (head0 + h) * p.S * D + d;
        const float* wh = wt + h * ns;
        float acc = 0.f;
        for (int k0 = 0; k0 < ns; k0 += 8) {  // eight slot loads in flight at a time
            float v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) v[u] = (k0 + u < ns) ? __ldcg(src + (size_t)(k0 + u) * D) : 0.f;
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (k0 + u < ns) acc += wh[k0 + u] * v[u];  // every written slot is finite
        }
        f.out[(head0 + h) * D + d] = __float2bfloat16(acc);
    }
    return consumer_sync(m, cph);  // the weights area is reused by the next run
}

template <int D, int BLK>
__device__ void step_consumers(const Params& p, const StepParams& f, const Smem& m) {
    using C = Cfg<D, BLK>;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tbase = warp * C::kTokPerWarp;  // this warp's token slice of each block
    int st = 0;
    uint32_t ph = 0, cph = 0;
    int cur_row = -1;
    WarpState<D, BLK> w;
    ws_reset(w);
    while (true) {
        const bool landed = mbar_wait(m.full(st), ph);
        __syncwarp();  // the lanes leave the wait together (ldmatrix / mma.sync below)
        if (!landed) {
            record_failure(m.info);
            break;
        }
        const volatile int* si = m.sinfo + st * kStageInfoWords;
        int sv[6];
#pragma unroll
        for (int i = 0; i < 6; ++i) sv[i] = si[i];  // read before the stage is released
        const int valid = sv[0], flags = sv[2];
        const uint32_t stK = m.sbase + (uint32_t)st * p.stage_bytes;
        if (flags & kExit) {
            __syncwarp();
            if (lane == 0) mbar_arrive(m.empty(st));
            break;
        }
        if (flags & kRunStart) {
            ws_reset(w);
            ws_load_q(w, reinterpret_cast<const __nv_bfloat16*>(m.base + (size_t)st * p.stage_bytes +
                                                                2 * C::kTileBytes),
                      p.G);
            cur_row = sv[1];
        }
        const bool wrote = (valid > tbase) && ws_block(w, stK, valid, tbase, p.G, p.scale_log2);
        if (wrote) fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(m.empty(st));
        if (++st == p.nst) {
            st = 0;
            ph ^= 1u;
        }
        if (flags & kRunEnd) {
            if (!step_flush<D, BLK>(p, f, m, w, sv, cph)) break;
            cur_row = -1;
        }
    }
    if (cur_row >= 0) {  // a wait gave up inside a run: the row's output shows it
        const int b = cur_row / p.Hkv, kvh = cur_row - b * p.Hkv;
        const size_t head0 = (size_t)b * p.Hq + (size_t)kvh * p.G;
        for (int idx = threadIdx.x; idx < p.G * D; idx += kConsumerThreads)
            f.out[head0 * D + idx] = __float2bfloat16(NAN);
    }
}

// ---------------------------------------------------------------- fused step: helper warps

// Decode phase, warps 9..11, beside the stream: refresh the pooled key of the
// open last block of every row whose last block lies in this CTA's gate range
// (one CTA per row). The gate never reads it (the last block is always kept),
// so it runs while the decode streams.
template <int D, int BLK>
__device__ void step_helpers(const Params& p, const StepParams& f, const Smem& m) {
    if ((int)blockIdx.x >= f.gate_ctas) return;
    PoolSmem<D>& psm = *reinterpret_cast<PoolSmem<D>*>(m.base + f.refresh_off);
    const int hwarp = ((int)threadIdx.x >> 5) - kHelperWarp0, lane = threadIdx.x & 31;
    const long long V1 = (long long)f.rows * f.NBmax;
    const long long h0 = (long long)blockIdx.x * V1 / f.gate_ctas;
    const long long h1 = (long long)(blockIdx.x + 1) * V1 / f.gate_ctas;
    uint32_t hph = 0;
    bool ok = true;
    auto hsync = [&]() {
        if (ok) ok = warp_group_sync(m.helper(), hph, m.info);
    };
    for (int gi = (int)(h0 / f.NBmax); ok && (long long)gi * f.NBmax < h1; ++gi) {
        const int r = gate_row(f, p.Hkv, gi);
        const int b = r / p.Hkv, kvh = r - b * p.Hkv;
        const int L = clamp_len(p.seq_lens[b], p.Lmax);
        const int NB = (L + BLK - 1) / BLK;
        if (NB == 0) continue;
        const long long last = (long long)gi * f.NBmax + NB - 1;
        if (last < h0 || last >= h1) continue;
        if (refresh_start_block(f, b, L, NB, BLK) > NB - 1) continue;
        const int j = NB - 1;
        pool_block_mean<D, BLK>(f.k_cache + ((size_t)r * p.Lmax + (size_t)j * BLK) * D, L - j * BLK, psm, hsync,
                                kHelperWarp0 * 32);
        float pv[D / 32];
#pragma unroll
        for (int u = 0; u < D / 32; ++u) pv[u] = psm.pooled[lane * (D / 32) + u];
        float* dst = f.kpool + ((size_t)r * f.NBmax + j) * f.dg;
        const float* W = f.w_k + (size_t)kvh * f.dg * D;
        warp_matvec_rows<D>(W, pv, hwarp, f.dg, kHelperThreads / 32, [&](int e, float x) { dst[e] = x; });
        hsync();  // the pool scratch is reused by the next row
    }
}

// kManyRows: rows outnumber the CTAs (the gate takes batches of rows, head-major);
// else one row per CTA. Two kernels, so neither mode's code shapes the other's.
template <int D, int BLK, int DG, bool kManyRows>
__global__ void __launch_bounds__(kStepThreads, 1)
    decode_step_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                       const Params p, const StepParams f) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const Smem m = setup_smem(smem_raw, p);
    unsigned long long old_ctr = 0;
    if (threadIdx.x == 0) {
        prefetch_tensor_map(&tmK);
        prefetch_tensor_map(&tmV);
        asm volatile("atom.add.relaxed.gpu.u64 %0, [%1], 1;" : "=l"(old_ctr) : "l"(f.launch_ctr) : "memory");
    }
    if (threadIdx.x == 0) {  // read after the gate's barriers
        SelList& sel = *reinterpret_cast<SelList*>(m.base + f.sel_off);
        sel.count = 0;
        sel.publish = -1;
        sel.early_count = 0;
        sel.thr_valid = 0;
    }
    gate_phase<D, BLK, DG, kManyRows>(&tmK, &tmV, p, f, m, old_ctr);
    fence_proxy_async_smem();  // the gate's use of the ring precedes the decode's copies into it
    if (threadIdx.x == 0) {
        const uint32_t epoch = epoch_of(old_ctr);
        m.info[kInfoEpoch] = (int)epoch;
        if (blockIdx.x == 0) f.rows_taken[(epoch + 1u) & 1u] = 0u;  // the next launch's tally
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5;
    if (warp == kConsumerWarps) {
        step_producer<D, BLK>(&tmK, &tmV, p, f, m);
    } else if (warp >= kHelperWarp0) {
        if (threadIdx.x == kHelperWarp0 * 32) {  // the row this CTA selected (rows fit the grid), after the barrier
            const int row = reinterpret_cast<const SelList*>(m.base + f.sel_off)->publish;
            if (row >= 0) st_release_u32(&f.rs[row].ready, (uint32_t)m.info[kInfoEpoch]);
        }
        __syncwarp();
        step_helpers<D, BLK>(p, f, m);
    } else {
        step_consumers<D, BLK>(p, f, m);
    }
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
    int nst, stage_bytes, merge_off, info_off, bar_off, refresh_off, sel_off, total;
};

template <int D, int BLK>
Layout make_layout(int G, bool with_refresh) {
    using C = Cfg<D, BLK>;
    Layout l;
    l.stage_bytes = (2 * C::kTileBytes + G * D * 2 + 1023) / 1024 * 1024;
    const int merge_bytes = max(kConsumerWarps * G * D * 4 + 2 * kConsumerWarps * G * 4,  // warp states
                                with_refresh ? kGateScratchBytes : 0);                   // or the gate's scratch
    const int info_bytes = (kInfoWords + kMaxStages * kStageInfoWords) * 4;
    const int bar_bytes = (2 * kMaxStages + 4 + kMaxGateStages) * 8;
    const int refresh_bytes = with_refresh ? (int)sizeof(PoolSmem<D>) + 16 : 0;
    const int sel_bytes = with_refresh ? (int)sizeof(SelList) : 0;
    const int tail = merge_bytes + info_bytes + bar_bytes + refresh_bytes + sel_bytes + 64;
    int nst = (kSmemLimit - 1024 - tail) / l.stage_bytes;
    l.nst = nst > kMaxStages ? kMaxStages : nst;
    l.merge_off = l.nst * l.stage_bytes;
    l.info_off = (l.merge_off + merge_bytes + 15) / 16 * 16;
    l.bar_off = (l.info_off + info_bytes + 15) / 16 * 16;
    l.refresh_off = l.bar_off + bar_bytes;
    l.sel_off = (l.refresh_off + refresh_bytes + 15) / 16 * 16;
    l.total = l.sel_off + sel_bytes + 1024;  // + slack for the 1024-byte alignment
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

// Raise a kernel's dynamic shared-memory ceiling once per device (the
// attribute belongs to each device's copy of the kernel).
template <typename K>
cudaError_t allow_big_smem(K kernel, bool (&done)[kMaxSmemDevices]) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < kMaxSmemDevices && done[dev]) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit);
    if (e == cudaSuccess && dev >= 0 && dev < kMaxSmemDevices) done[dev] = true;  // benign race: set twice
    return e;
}

template <int D, int BLK>
cudaError_t launch_impl(const Shape& s, const DecodeLaunch& a, const CUtensorMap& tmK, const CUtensorMap& tmV,
                        int num_sms, cudaStream_t stream) {
    const Layout l = make_layout<D, BLK>(s.G, false);
    if (l.nst < 2) return cudaErrorInvalidConfiguration;
    static bool attr_done[kMaxSmemDevices] = {};
    cudaError_t e = allow_big_smem(sparse_decode_kernel<D, BLK>, attr_done);
    if (e != cudaSuccess) return e;
    const Params p = make_params<D, BLK>(s, a, l, sparse_decode_ctas(s, a.kmax, a.num_splits, num_sms));
    return launch_after_prior(sparse_decode_kernel<D, BLK>, dim3(p.P), dim3(kThreads), l.total, stream, nullptr, tmK,
                              tmV, p);
}

// How the fused step spreads its work (the same on the host and in the workspace layout).
struct StepGeometry {
    int gate_ctas;  // CTAs of the gate
    int gate_cpr;   // CTAs per row when rows fit the grid, else 0
    int chunk;      // list positions per claim
    int nslots;     // partial slots per (row, head): one per chunk
};

StepGeometry step_geometry(const Shape& s, int kmax, int num_sms) {
    StepGeometry g;
    const long long rows = (long long)s.B * s.Hkv;
    if (rows <= num_sms) {
        const int per_row = (int)(num_sms / rows);
        const int cap = (s.NBmax + kMinGatePositions - 1) / kMinGatePositions;
        g.gate_cpr = per_row < cap ? per_row : cap;
        if (g.gate_cpr < 1) g.gate_cpr = 1;
        g.gate_ctas = (int)rows * g.gate_cpr;
    } else {
        g.gate_cpr = 0;
        g.gate_ctas = num_sms;
    }
    // about 64 KB of K+V per claim, at most 64 claims per row. A run holds at
    // least one whole chunk except the front and the back piece that meet, so
    // a row has at most chunks + 2 runs, each with its slot; with fixed parts
    // (rows fit the grid) a row has min(kmax, CTAs per row) non-empty parts.
    const int base = s.blk == 64 ? 2 : 1;
    const int c = (kmax + 63) / 64;
    g.chunk = c < base ? base : c;
    g.nslots = (kmax + g.chunk - 1) / g.chunk + 2;
    const int parts = kmax < g.gate_cpr ? kmax : g.gate_cpr;
    if (parts > g.nslots) g.nslots = parts;
    return g;
}

template <int D, int BLK, int DG>
cudaError_t step_impl(const Shape& s, const StepLaunch& a, const CUtensorMap& tmK, const CUtensorMap& tmV,
                      int num_sms, cudaStream_t stream) {
    const Layout l = make_layout<D, BLK>(s.G, true);
    if (l.nst < 2) return cudaErrorInvalidConfiguration;
    const int keys_bytes = (s.NBmax * 4 + 1023) / 1024 * 1024;
    const int ring = l.nst * l.stage_bytes;
    const int n_gate = (ring - keys_bytes) / kGateChunkBytes;
    if (n_gate < 1) return cudaErrorInvalidConfiguration;
    static bool attr_done[kMaxSmemDevices] = {};
    static bool attr_done_many[kMaxSmemDevices] = {};
    cudaError_t e = allow_big_smem(decode_step_kernel<D, BLK, DG, false>, attr_done);
    if (e == cudaSuccess) e = allow_big_smem(decode_step_kernel<D, BLK, DG, true>, attr_done_many);
    if (e != cudaSuccess) return e;
    const int kmax = a.budget_tokens / s.blk;
    const StepGeometry geo = step_geometry(s, kmax, num_sms);
    unsigned char* ws = static_cast<unsigned char*>(a.workspace);
    const WorkspaceLayout wl = step_workspace_layout(s, kmax, num_sms);

    DecodeLaunch d;
    d.q = a.q;
    d.seq_lens = a.seq_lens;
    d.block_idx = a.block_idx;
    d.num_selected = a.num_selected;
    d.o_part = reinterpret_cast<float*>(ws + wl.o_part);
    d.lse_part = reinterpret_cast<float*>(ws + wl.lse_part);
    d.kmax = kmax;
    d.num_splits = geo.nslots;
    d.sm_scale = a.sm_scale;
    const Params p = make_params<D, BLK>(s, d, l, num_sms);

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
    f.launch_ctr = reinterpret_cast<unsigned long long*>(ws + wl.launch_ctr);
    f.rows_taken = reinterpret_cast<unsigned int*>(ws + wl.rows_taken);
    f.row_cnt = reinterpret_cast<unsigned int*>(ws + wl.row_cnt);
    f.rs = reinterpret_cast<RowState*>(ws + wl.row_state);
    f.keys_g = reinterpret_cast<uint32_t*>(ws + wl.keys);
    f.rows = s.B * s.Hkv;
    f.gate_ctas = geo.gate_ctas;
    f.gate_cpr = geo.gate_cpr;
    f.chunk = geo.chunk;
    f.NBmax = s.NBmax;
    f.dg = s.dg;
    f.refresh_off = l.refresh_off;
    f.sel_off = l.sel_off;
    f.keys_off = ring - keys_bytes;  // the gate's order keys end the ring: the early stages start at its front
    f.chunk_off = 0;
    f.n_gate_stages = n_gate > kMaxGateStages ? kMaxGateStages : n_gate;
    // one CTA per row: decode stages that fit before the keys may start during the selection
    const int n_early = f.keys_off / l.stage_bytes < l.nst - 1 ? f.keys_off / l.stage_bytes : l.nst - 1;
    f.n_early = geo.gate_cpr == 1 ? n_early : 0;
    // W_q of a batch's head (dg x D fp32; one row per CTA, or rows outnumbering the CTAs
    // taken head-major) first fills the last gate stages
    const int wq_st = (DG * D * 4 + kGateChunkBytes - 1) / kGateChunkBytes;
    f.wq_stages = f.n_gate_stages > wq_st ? wq_st : 0;

    // One CTA per SM, all co-resident (the decode phase waits on rows that other CTAs publish).
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(num_sms, 1, 1);
    cfg.blockDim = dim3(kStepThreads, 1, 1);
    cfg.dynamicSmemBytes = l.total;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = geo.gate_cpr > 0 ? cudaLaunchKernelEx(&cfg, decode_step_kernel<D, BLK, DG, false>, tmK, tmV, p, f)
                         : cudaLaunchKernelEx(&cfg, decode_step_kernel<D, BLK, DG, true>, tmK, tmV, p, f);
    if (e != cudaSuccess) (void)cudaGetLastError();  // a rejected launch must not leak into the next call
    return e;
}

}  // namespace

WorkspaceLayout step_workspace_layout(const Shape& s, int kmax, int num_sms) {
    WorkspaceLayout w;
    const size_t rows = (size_t)s.B * s.Hkv;
    const size_t S = (size_t)step_geometry(s, kmax, num_sms).nslots;
    auto up = [](size_t x) { return (x + 255) / 256 * 256; };
    w.launch_ctr = 0;
    w.rows_taken = 8;
    w.row_cnt = 256;
    w.row_state = up(w.row_cnt + rows * 4);
    w.counters_end = up(w.row_state + rows * sizeof(RowState));  // everything before this must start at zero
    w.keys = w.counters_end;
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
    // The array keeps the previous call's contents: the launch counter, the
    // row states and the gate counts must start at zero.
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
