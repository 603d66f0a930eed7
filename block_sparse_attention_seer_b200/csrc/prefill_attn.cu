// prefill_attn.cu -- causal block-sparse attention of a prompt on the
// fifth-generation tensor cores (tcgen05, accumulators in tensor memory).
//
// Computes, for token t of query block i (head h of KV group kvh, sequence
// b), softmax attention over the tokens u <= t, u < L_b, of the key blocks
// kept for (b, kvh, i): the block-sparse FlashAttention step of
// "SeerAttention: Learning Intrinsic Sparse Attention in Your LLMs"
// (abstract), with the gate's kept blocks as the sparsity pattern.
//
// Design (one CTA per (b, kvh, query block, group of heads)):
//  * the CTA's query rows -- up to 256: the heads of the group that share
//    the kept blocks, BLK rows each -- form two M = 128 tiles whose Q stays
//    in shared memory. The kept key blocks are walked as 128-key sub-tiles
//    (two kept 64-token blocks, or one 128-token block; the MMA does not care
//    that the two halves are apart in the cache), so one K/V copy serves every
//    head of the group and each MMA has N = 128;
//  * warp 8, one lane: TMA producer (2-D tiles, 128-byte swizzle) of Q once
//    and of K and V through separate rings (K is released as soon as both S
//    tiles have read it, V after both P V);
//  * warp 9, one lane: issues the MMAs in the order P V_0(n), S_0(n+1),
//    P V_1(n), S_1(n+1), so the tensor core computes one tile while the other
//    tile's softmax runs. S_t = Q_t K^T (M 128, N 128, K D) lands in TMEM; the
//    softmax writes P_t as bf16 pairs over the upper 64 of its 128 columns
//    (already read into registers); O_t += P_t V takes P_t straight from
//    TMEM (A operand in tensor memory) -- no P round trip through shared
//    memory, which would cost operand bandwidth;
//  * warps 0-3 and 4-7: one softmax warpgroup per tile, a thread per row
//    (TMEM lane): reads its S row, masks (causal on the diagonal block, the
//    sequence end, an absent second half), online softmax in the exp2 domain
//    with a lazily moved reference maximum (O and l are rescaled in TMEM only
//    when the row maximum grows by more than 2^8; the max is three-input
//    max.f32, the scale-subtract and the row sum paired fp32 instructions),
//    writes P; at the end reads O, divides by l and stores the row;
//  * every wait is bounded; on expiry the CTA stops, drains its own copies and
//    MMAs, frees its tensor memory and writes NaN rows.
#include <cuda_bf16.h>

#include <cmath>

#include "seer_device.cuh"
#include "seer_launch.h"
#include "tcgen05.cuh"

namespace seer {
namespace {

constexpr int kAttnThreads = 320;   // 8 softmax warps, producer, MMA
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kRowsPerCta = 256;    // two M = 128 tiles
constexpr int kHalf = 64;           // key tokens per half sub-tile (one TMA box of rows)
constexpr int kSub = 128;           // key tokens per sub-tile
constexpr int kTmemCols = 512;      // per tile: O at +0 (D columns), S at +128 (128 columns), P at +192
constexpr int kSCol = 128;
constexpr int kAttnSmemLimit = 232448;
constexpr float kLog2eA = 1.44269504088896340736f;
constexpr float kLn2A = 0.69314718055994530942f;
constexpr float kRescaleLog2 = 8.0f;  // move the reference maximum only past a 2^8 growth
constexpr int kListCap = 384;         // kept lists up to this length are staged in shared memory

template <int D>
struct AttnCfg {
    static constexpr int kBoxes = D / 64;                // 128-byte column boxes of a row
    static constexpr int kQTile = kBoxes * 128 * 128;    // one M tile of Q
    static constexpr int kBox = kSub * 128;              // one column box of a K or V sub-tile
    static constexpr int kKV = kBoxes * kBox;            // K (or V) of one sub-tile
    static constexpr int kBarBytes = 256 + kListCap * 4;
    static constexpr int kRing = (kAttnSmemLimit - 1024 - kBarBytes - 2 * kQTile) / kKV;  // K + V slots
    // a V slot is held from its copy until both P V have read it, a K slot only
    // until both S have: V gets the deeper ring
    static constexpr int kKSt = kRing >= 8 ? 4 : 2;
    static constexpr int kVSt = kRing - kKSt > 6 ? 6 : kRing - kKSt;
    static constexpr int kSmem = 1024 + 2 * kQTile + (kKSt + kVSt) * kKV + kBarBytes;
    static_assert(kVSt >= 2 && kKSt >= 2, "too little shared memory for the K/V rings");
    static_assert(D <= kSCol && kSCol + kSub <= kTmemCols / 2, "TMEM columns of one tile");
};

// The kept (b, kvh, i) list walked as sub-tiles of two 64-token halves:
// entries outside [0, i] are skipped; with 64-token blocks a sub-tile takes
// two consecutive kept blocks (the last one may have one), with 128-token
// blocks one block, its second half absent when it starts at or past L.
struct PairIter {
    const int32_t* list;
    int nsel, i, L, blk;
    int x;            // next list position
    int tokA, tokB;   // token bases of the halves; tokB < 0: absent
    bool valid;
    __device__ int next_entry() {
        while (x < nsel) {
            const int j = list[x++];
            if (j >= 0 && j <= i && j * blk < L) return j;
        }
        return -1;
    }
    __device__ void advance() {
        const int ja = next_entry();
        valid = ja >= 0;
        if (!valid) return;
        tokA = ja * blk;
        if (blk == kSub) {
            tokB = tokA + kHalf < L ? tokA + kHalf : -1;
        } else {
            const int jb = next_entry();
            tokB = jb >= 0 ? jb * blk : -1;
        }
    }
    __device__ void start() {
        x = 0;
        advance();
    }
};

struct AttnBars {
    uint32_t q_full, k_full, k_empty, v_full, v_empty, s_ready, p_ready, o_done, drain;
    // k_* : + 8 * slot, v_* : + 8 * slot; s_ready / p_ready / o_done: + 8 * tile
};

// 2^x on the special-function unit (flush-to-zero; 2^-inf = 0).
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// max of three (one instruction on sm_100)
__device__ __forceinline__ float fmax3f(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// P for 64 scores of a row: 2^(s * scale + neg_m) as bf16 pairs into 32 TMEM
// columns from `taddr` (paired fp32 FMA and add); the row sum goes to sum2.
__device__ __forceinline__ void emit_p(const uint32_t (&sh)[2][32], float scale_log2, float neg_m, float2 (&sum2)[2],
                                       uint32_t taddr) {
    const float2 sc = make_float2(scale_log2, scale_log2), nm = make_float2(neg_m, neg_m);
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const float2 x = __ffma2_rn(make_float2(__uint_as_float(sh[q][2 * e]), __uint_as_float(sh[q][2 * e + 1])),
                                        sc, nm);
            const float2 pp = make_float2(ex2(x.x), ex2(x.y));
            sum2[e & 1] = __fadd2_rn(sum2[e & 1], pp);
            pk[e] = pack_bf16x2(pp.x, pp.y);
        }
        tc::st_32x32b_x16(taddr + (uint32_t)(16 * q), pk);
    }
}

__device__ __forceinline__ bool abort_set(const int* flag) { return *(volatile const int*)flag != 0; }

template <int D, int BLK>
__global__ void __launch_bounds__(kAttnThreads, 1)
    prefill_attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                           const __grid_constant__ CUtensorMap tmV, const int32_t* __restrict__ seq_lens,
                           const int32_t* __restrict__ block_idx, const int32_t* __restrict__ num_selected, int Hq,
                           int Hkv, int Lmax, int NBmax, int kmax, int heads_per_cta, int n_hsplit,
                           float scale_log2, __nv_bfloat16* __restrict__ out, float* __restrict__ lse_out) {
    using C = AttnCfg<D>;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = Hq / Hkv;
    const int i = NBmax - 1 - (int)(blockIdx.x / n_hsplit);  // the longest rows first
    const int hs = (int)(blockIdx.x % n_hsplit);
    const int row = blockIdx.y;
    const int b = row / Hkv, kvh = row - b * Hkv;
    const int h0 = kvh * G + hs * heads_per_cta;              // first query head of this CTA
    const int nh = min(heads_per_cta, G - hs * heads_per_cta);
    const int nrows = nh * BLK;
    const int n_tiles = (nrows + 127) / 128;
    const int L = clamp_len(seq_lens[b], Lmax);
    const int t0 = i * BLK;

    // a query block wholly past the length: zero rows, lse -inf
    if (t0 >= L) {
        for (int x = tid; x < nrows * (D / 8); x += kAttnThreads) {
            const int r = x / (D / 8), c = x - r * (D / 8);
            const int hl = r / BLK, t = t0 + (r - hl * BLK);
            if (t < Lmax)
                *reinterpret_cast<uint4*>(out + ((size_t)(b * Hq + h0 + hl) * Lmax + t) * D + c * 8) =
                    make_uint4(0u, 0u, 0u, 0u);
        }
        if (lse_out)
            for (int r = tid; r < nrows; r += kAttnThreads) {
                const int hl = r / BLK, t = t0 + (r - hl * BLK);
                if (t < Lmax) lse_out[(size_t)(b * Hq + h0 + hl) * Lmax + t] = -INFINITY;
            }
        return;
    }

    // ---- shared memory: Q tiles, K ring, V ring, barriers, kept list
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char* gbase = smem_raw + (base - raw);
    const uint32_t sQ = base, sK = base + 2 * C::kQTile, sV = sK + C::kKSt * C::kKV;
    const uint32_t sBar = sV + C::kVSt * C::kKV;
    unsigned char* gBar = gbase + (sBar - base);
    AttnBars bars;
    bars.q_full = sBar;
    bars.k_full = sBar + 8;
    bars.k_empty = bars.k_full + 8 * C::kKSt;
    bars.v_full = bars.k_empty + 8 * C::kKSt;
    bars.v_empty = bars.v_full + 8 * C::kVSt;
    bars.s_ready = bars.v_empty + 8 * C::kVSt;
    bars.p_ready = bars.s_ready + 8 * 2;
    bars.o_done = bars.p_ready + 8 * 2;
    bars.drain = bars.o_done + 8 * 2;
    const uint32_t bar_end = bars.drain + 8;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gBar + (bar_end - sBar));
    int* abort_flag = reinterpret_cast<int*>(gBar + (bar_end - sBar) + 4);
    int32_t* list_s = reinterpret_cast<int32_t*>(gBar + 256);

    if (tid == 0) {
        mbar_init(bars.q_full, 1);
        for (int s = 0; s < C::kKSt; ++s) {
            mbar_init(bars.k_full + 8 * s, 1);
            mbar_init(bars.k_empty + 8 * s, 1);
        }
        for (int s = 0; s < C::kVSt; ++s) {
            mbar_init(bars.v_full + 8 * s, 1);
            mbar_init(bars.v_empty + 8 * s, 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(bars.s_ready + 8 * t, 1);
            mbar_init(bars.p_ready + 8 * t, 4);
            mbar_init(bars.o_done + 8 * t, 1);
        }
        mbar_init(bars.drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        tc::tmem_alloc(smem_addr(tmem_slot), kTmemCols);
        tc::tmem_relinquish();
    }
    const int32_t* list_g = block_idx + ((size_t)row * NBmax + i) * kmax;
    const int nsel = min(max(num_selected[(size_t)row * NBmax + i], 0), kmax);
    for (int x = tid; x < nsel && nsel <= kListCap; x += kAttnThreads) list_s[x] = list_g[x];
    const int32_t* list = nsel <= kListCap ? list_s : list_g;
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_slot);

    PairIter it0;
    it0.list = list;
    it0.nsel = nsel;
    it0.i = i;
    it0.L = L;
    it0.blk = BLK;
    it0.start();
    const bool any = it0.valid;

    auto fail = [&]() { atomicExch(abort_flag, 1); };

    if (warp == kProducerWarp) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0 && any) {
            prefetch_tensor_map(&tmQ);
            prefetch_tensor_map(&tmK);
            prefetch_tensor_map(&tmV);
            const uint64_t pol = l2_policy_evict_first();
            mbar_arrive_expect_tx(bars.q_full, (uint32_t)(nrows * D * 2));
            for (int hl = 0; hl < nh; ++hl) {
                const int r0 = hl * BLK;  // CTA row of the head's first query
                const uint32_t dst = sQ + (r0 / 128) * C::kQTile + (r0 % 128) * 128;
                const int y = (b * Hq + h0 + hl) * Lmax + t0;
                for (int c = 0; c < C::kBoxes; ++c) tma_load_2d(dst + c * 128 * 128, &tmQ, bars.q_full, c * 64, y, pol);
            }
            // K/V tiles are re-read by the other query blocks of the row: keep them in L2
            uint64_t keep;
            asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(keep));
            PairIter it = it0;
            int n = 0;
            bool ok = true;
            for (; it.valid; it.advance(), ++n) {
                const int halves = it.tokB >= 0 ? 2 : 1;
                const uint32_t bytes = (uint32_t)(halves * C::kBoxes * kHalf * 128);
                const int ks = n % C::kKSt, vs = n % C::kVSt;
                if (n >= C::kKSt && !mbar_wait(bars.k_empty + 8 * ks, (uint32_t)((n / C::kKSt - 1) & 1))) ok = false;
                if (!ok || abort_set(abort_flag)) break;
                mbar_arrive_expect_tx(bars.k_full + 8 * ks, bytes);
                for (int h = 0; h < halves; ++h) {
                    const int y = row * Lmax + (h == 0 ? it.tokA : it.tokB);
                    for (int c = 0; c < C::kBoxes; ++c)
                        tma_load_2d(sK + ks * C::kKV + c * C::kBox + h * kHalf * 128, &tmK, bars.k_full + 8 * ks,
                                    c * 64, y, keep);
                }
                if (n >= C::kVSt && !mbar_wait(bars.v_empty + 8 * vs, (uint32_t)((n / C::kVSt - 1) & 1))) ok = false;
                if (!ok || abort_set(abort_flag)) {
                    ++n;  // the K copies of this sub-tile are in flight
                    break;
                }
                mbar_arrive_expect_tx(bars.v_full + 8 * vs, bytes);
                for (int h = 0; h < halves; ++h) {
                    const int y = row * Lmax + (h == 0 ? it.tokA : it.tokB);
                    for (int c = 0; c < C::kBoxes; ++c)
                        tma_load_2d(sV + vs * C::kKV + c * C::kBox + h * kHalf * 128, &tmV, bars.v_full + 8 * vs,
                                    c * 64, y, keep);
                }
            }
            if (!ok) fail();
            // leave only after the copies issued have landed
            const int issued = n;
            for (int m = max(0, issued - C::kKSt); m < issued; ++m)
                (void)mbar_wait(bars.k_full + 8 * (m % C::kKSt), (uint32_t)((m / C::kKSt) & 1));
            for (int m = max(0, issued - C::kVSt); m < issued; ++m)
                (void)mbar_wait(bars.v_full + 8 * (m % C::kVSt), (uint32_t)((m / C::kVSt) & 1));
            (void)mbar_wait(bars.q_full, 0u);
        }
        __syncwarp();
    }
    else if (warp == kMmaWarp) {
        // ---------------------------------------------------------------- MMA issue
        if (lane == 0 && any) {
            constexpr uint32_t kIdS = tc::idesc_bf16_f32(128, kSub, false);
            constexpr uint32_t kIdO = tc::idesc_bf16_f32(128, D, true);
            bool ok = mbar_wait(bars.q_full, 0u);
            const uint64_t dq0 = tc::smem_desc_sw128(sQ, 16, 1024);
            const uint64_t dq1 = tc::smem_desc_sw128(sQ + C::kQTile, 16, 1024);
            // S_t(n) = Q_t K(n)^T into the tile's S columns; the k-th 16-column step
            // is box k / 4, 32 bytes * (k % 4) into each swizzled 128-byte row
            auto issue_s = [&](int t, int n) {
                const uint64_t dk = tc::smem_desc_sw128(sK + (n % C::kKSt) * C::kKV, 16, 1024);
                const uint64_t dq = t == 0 ? dq0 : dq1;
                const uint32_t d_tmem = tmem + (uint32_t)(t * (kTmemCols / 2) + kSCol);
#pragma unroll
                for (int k = 0; k < D / 16; ++k)
                    tc::mma_bf16_ss(d_tmem, dq + (uint64_t)((k >> 2) * (128 * 128 / 16) + (k & 3) * 2),
                                    dk + (uint64_t)((k >> 2) * (C::kBox / 16) + (k & 3) * 2), kIdS, k > 0);
                tc::commit(bars.s_ready + 8 * t);
            };
            if (ok) ok = mbar_wait(bars.k_full, 0u);  // K(0): slot 0, first phase
            if (ok) {
                tc::fence_after_sync();
                for (int t = 0; t < n_tiles; ++t) issue_s(t, 0);
                tc::commit(bars.k_empty);  // slot 0 is free once both S(0) are done
            }
            PairIter it = it0;
            int n = 0;
            while (ok && it.valid) {
                PairIter nx = it;
                nx.advance();
                const bool more = nx.valid;
                const int vs = n % C::kVSt, ks1 = (n + 1) % C::kKSt;
                const int ksteps = it.tokB >= 0 ? kSub / 16 : kHalf / 16;  // an absent half is skipped
                if (!mbar_wait(bars.v_full + 8 * vs, (uint32_t)((n / C::kVSt) & 1)) ||
                    (more && !mbar_wait(bars.k_full + 8 * ks1, (uint32_t)(((n + 1) / C::kKSt) & 1)))) {
                    ok = false;
                    break;
                }
                // V: MN-major (keys x D); the k-th 16-key step is 16 rows further, the
                // next 64 columns of D one box further (leading byte offset)
                const uint64_t dv = tc::smem_desc_sw128(sV + vs * C::kKV, C::kBox, 1024);
                for (int t = 0; t < n_tiles; ++t) {
                    if (!mbar_wait(bars.p_ready + 8 * t, (uint32_t)(n & 1))) {
                        ok = false;
                        break;
                    }
                    tc::fence_after_sync();
                    const uint32_t o_tmem = tmem + (uint32_t)(t * (kTmemCols / 2));
                    for (int k = 0; k < ksteps; ++k)
                        tc::mma_bf16_ts(o_tmem, o_tmem + (uint32_t)(kSCol + 64 + k * 8),
                                        dv + (uint64_t)(k * (16 * 128 / 16)), kIdO, n > 0 || k > 0);
                    // S_t(n+1) overwrites P_t(n) only after P V_t(n) has read it: the tensor
                    // core runs one thread's MMAs in issue order
                    if (more) issue_s(t, n + 1);
                }
                if (!ok) break;
                tc::commit(bars.v_empty + 8 * vs);           // V(n) read by every P V
                if (more) tc::commit(bars.k_empty + 8 * ks1);  // K(n+1) read by every S
                if (abort_set(abort_flag)) {
                    ok = false;
                    break;
                }
                it = nx;
                ++n;
            }
            if (!ok) fail();
            for (int t = 0; t < n_tiles; ++t) tc::commit(bars.o_done + 8 * t);
            // every MMA issued has completed before the tensor memory is freed
            tc::commit(bars.drain);
            (void)mbar_wait(bars.drain, 0u);
        }
        __syncwarp();
    } else if (warp / 4 < n_tiles && any) {
        // ---------------------------------------------------------------- softmax, one row per thread
        const int t = warp / 4;
        const int r = (warp & 3) * 32 + lane;       // TMEM lane = row of the tile
        const int lr = t * 128 + r;                  // CTA row
        const int hl = lr / BLK;
        const bool real = hl < nh;
        const int qt = t0 + (lr - hl * BLK);         // query token
        const int lim_tok = min(qt, L - 1);          // last key token this row may see
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t t_tmem = tmem + lane_base + (uint32_t)(t * (kTmemCols / 2));
        float m_ref = -INFINITY, l = 0.f;
        bool ok = true;
        PairIter it = it0;
        int n = 0;
        for (; it.valid; it.advance(), ++n) {
            const bool w = mbar_wait(bars.s_ready + 8 * t, (uint32_t)(n & 1));
            if (__any_sync(0xffffffffu, !w || abort_set(abort_flag))) {  // one decision for the warp
                ok = false;
                break;
            }
            tc::fence_after_sync();
            // mask (only the diagonal, the sequence end, an absent half)
            const int limA = lim_tok - it.tokA;
            const int limB = it.tokB >= 0 ? lim_tok - it.tokB : -1;
            const bool masked = !__all_sync(0xffffffffu, limA >= kHalf - 1 && limB >= kHalf - 1);
            // half A (keys 0-63): its maximum only; half B (keys 64-127) stays in registers
            uint32_t sh[2][32];
            tc::ld_32x32b_x32(t_tmem + (uint32_t)kSCol, sh[0]);
            tc::ld_32x32b_x32(t_tmem + (uint32_t)(kSCol + 32), sh[1]);
            tc::wait_ld();
            if (masked) {
#pragma unroll
                for (int c = 0; c < kHalf; ++c)
                    if (c > limA) sh[c >> 5][c & 31] = __float_as_uint(-INFINITY);
            }
            float m8[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) m8[e] = -INFINITY;
#pragma unroll
            for (int c = 0; c < kHalf; c += 2)
                m8[(c >> 1) & 7] = fmax3f(m8[(c >> 1) & 7], __uint_as_float(sh[c >> 5][c & 31]),
                                          __uint_as_float(sh[c >> 5][(c + 1) & 31]));
            tc::ld_32x32b_x32(t_tmem + (uint32_t)(kSCol + 64), sh[0]);
            tc::ld_32x32b_x32(t_tmem + (uint32_t)(kSCol + 96), sh[1]);
            tc::wait_ld();
            if (masked) {
#pragma unroll
                for (int c = 0; c < kHalf; ++c)
                    if (c > limB) sh[c >> 5][c & 31] = __float_as_uint(-INFINITY);
            }
#pragma unroll
            for (int c = 0; c < kHalf; c += 2)
                m8[(c >> 1) & 7] = fmax3f(m8[(c >> 1) & 7], __uint_as_float(sh[c >> 5][c & 31]),
                                          __uint_as_float(sh[c >> 5][(c + 1) & 31]));
            const float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                                   fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7]))) * scale_log2;  // scale > 0
            float alpha = 1.f;
            if (mx > m_ref + kRescaleLog2 || (m_ref == -INFINITY && mx > -INFINITY)) {
                alpha = m_ref == -INFINITY ? 0.f : ex2(m_ref - mx);
                m_ref = mx;
                l *= alpha;
            }
            // P = 2^(s * scale - m) as bf16 pairs over the upper 64 S columns (keys 64-127 read
            // already): half B into columns +96.., then half A, read again, into +64..
            const float neg_m = m_ref == -INFINITY ? 0.f : -m_ref;
            float2 sum2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
            auto emit = [&](int col) { emit_p(sh, scale_log2, neg_m, sum2, t_tmem + (uint32_t)col); };
            emit(kSCol + 96);
            // O_t is final up to P V_t(n-1) (issued before S_t(n)): rescale it if needed
            if (n > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
                for (int c0 = 0; c0 < D; c0 += 32) {
                    uint32_t o[32];
                    tc::ld_32x32b_x32(t_tmem + (uint32_t)c0, o);
                    tc::wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                    tc::st_32x32b_x32(t_tmem + (uint32_t)c0, o);
                }
            }
            tc::ld_32x32b_x32(t_tmem + (uint32_t)kSCol, sh[0]);
            tc::ld_32x32b_x32(t_tmem + (uint32_t)(kSCol + 32), sh[1]);
            tc::wait_ld();
            if (masked) {
#pragma unroll
                for (int c = 0; c < kHalf; ++c)
                    if (c > limA) sh[c >> 5][c & 31] = __float_as_uint(-INFINITY);
            }
            emit(kSCol + 64);
            l += (sum2[0].x + sum2[0].y) + (sum2[1].x + sum2[1].y);
            tc::wait_st();
            // the sequence end inside a half: zero its V rows past L (they may hold anything)
            if (t == 0) {
                const int vA = it.tokA + kHalf > L ? L - it.tokA : kHalf;
                const int vB = it.tokB >= 0 && it.tokB + kHalf > L ? L - it.tokB : kHalf;
                if (vA < kHalf || vB < kHalf) {
                    const int vs = n % C::kVSt;
                    const bool wv = mbar_wait(bars.v_full + 8 * vs, (uint32_t)((n / C::kVSt) & 1));
                    if (!wv) fail();
                    const uint32_t sv = sV + vs * C::kKV;
                    for (int h = 0; h < 2; ++h) {
                        const int v0 = h == 0 ? vA : vB;
                        for (int x = (warp & 3) * 32 + lane; x < (kHalf - v0) * C::kBoxes * 8; x += 128) {
                            const int rr = h * kHalf + v0 + x / (C::kBoxes * 8), rem = x % (C::kBoxes * 8);
                            const uint32_t a = sv + (rem >> 3) * C::kBox + rr * 128 + (rem & 7) * 16;
                            asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(0u) : "memory");
                        }
                    }
                    fence_proxy_async_smem();
                }
            }
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(bars.p_ready + 8 * t);
        }
        // ---- epilogue: O / l
        if (ok) {
            const bool w = mbar_wait(bars.o_done + 8 * t, 0u);
            if (__any_sync(0xffffffffu, !w)) ok = false;
            tc::fence_after_sync();
        }
        if (!ok) fail();
        const bool write = real && qt < Lmax;
        const bool valid = ok && qt < L && l > 0.f;
        const float inv = valid ? 1.f / l : 0.f;
        const int h = h0 + hl;
        __nv_bfloat16* orow = out + ((size_t)(b * Hq + h) * Lmax + qt) * D;
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t o[32];
            tc::ld_32x32b_x32(t_tmem + (uint32_t)c0, o);
            tc::wait_ld();
            if (write) {
                uint32_t pkd[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float a0 = ok ? __uint_as_float(o[2 * e]) * inv : NAN;
                    const float a1 = ok ? __uint_as_float(o[2 * e + 1]) * inv : NAN;
                    pkd[e] = (qt < L || !ok) ? pack_bf16x2(a0, a1) : 0u;
                }
#pragma unroll
                for (int v = 0; v < 4; ++v)
                    *reinterpret_cast<uint4*>(orow + c0 + 8 * v) =
                        make_uint4(pkd[4 * v], pkd[4 * v + 1], pkd[4 * v + 2], pkd[4 * v + 3]);
            }
        }
        if (write && lse_out)
            lse_out[(size_t)(b * Hq + h) * Lmax + qt] =
                !ok ? NAN : (valid ? (m_ref + log2f(l)) * kLn2A : -INFINITY);
        tc::fence_before_sync();
    } else if (warp / 4 < n_tiles) {
        // no kept block at all: zero rows, lse -inf
        const int t = warp / 4, r = (warp & 3) * 32 + lane, lr = t * 128 + r, hl = lr / BLK;
        const int qt = t0 + (lr - hl * BLK);
        if (hl < nh && qt < Lmax) {
            __nv_bfloat16* orow = out + ((size_t)(b * Hq + h0 + hl) * Lmax + qt) * D;
            for (int c = 0; c < D; c += 8) *reinterpret_cast<uint4*>(orow + c) = make_uint4(0u, 0u, 0u, 0u);
            if (lse_out) lse_out[(size_t)(b * Hq + h0 + hl) * Lmax + qt] = -INFINITY;
        }
    }
    __syncthreads();
    if (warp == kMmaWarp) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

template <int D, int BLK>
cudaError_t attn_tc_impl(const Shape& s, const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                         const int32_t* seq_lens, const int32_t* block_idx, const int32_t* num_selected, int kmax,
                         float sm_scale, void* out, float* lse_out, cudaStream_t stream) {
    using C = AttnCfg<D>;
    static bool attr_done = false;
    if (!attr_done) {
        const cudaError_t e = cudaFuncSetAttribute(prefill_attn_tc_kernel<D, BLK>,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
        if (e != cudaSuccess) return e;
        attr_done = true;
    }
    const int heads_per_cta = s.G < kRowsPerCta / BLK ? s.G : kRowsPerCta / BLK;
    const int n_hsplit = (s.G + heads_per_cta - 1) / heads_per_cta;
    const dim3 grid((unsigned)(s.NBmax * n_hsplit), (unsigned)(s.B * s.Hkv));
    prefill_attn_tc_kernel<D, BLK><<<grid, kAttnThreads, C::kSmem, stream>>>(
        tmQ, tmK, tmV, seq_lens, block_idx, num_selected, s.Hq, s.Hkv, s.Lmax, s.NBmax, kmax, heads_per_cta,
        n_hsplit, sm_scale * kLog2eA, static_cast<__nv_bfloat16*>(out), lse_out);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_attention(const Shape& s, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                                     const CUtensorMap& tmV, const int32_t* seq_lens, const int32_t* block_idx,
                                     const int32_t* num_selected, int kmax, float sm_scale, void* out, float* lse_out,
                                     cudaStream_t stream) {
#define SEER_ATTN_CASE(DV, BV)                                                                                    \
    if (s.D == DV && s.blk == BV)                                                                                 \
        return attn_tc_impl<DV, BV>(s, tmQ, tmK, tmV, seq_lens, block_idx, num_selected, kmax, sm_scale, out,    \
                                    lse_out, stream);
    SEER_ATTN_CASE(128, 64)
    SEER_ATTN_CASE(128, 128)
    SEER_ATTN_CASE(64, 64)
    SEER_ATTN_CASE(64, 128)
#undef SEER_ATTN_CASE
    return cudaErrorInvalidValue;
}

}  // namespace seer
