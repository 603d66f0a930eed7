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
//    in shared memory; every kept key block is walked as 64-token sub-tiles,
//    so one K/V copy serves every head of the group;
//  * warp 8, one lane: TMA producer (2-D tiles, 128-byte swizzle) of Q once
//    and of K/V sub-tiles through a ring of stages;
//  * warp 9, one lane: issues the MMAs. S_t = Q_t K^T (M 128, N 64, K D) into
//    a double-buffered TMEM tile, then O_t += P_t V (M 128, N D, K 64) into a
//    TMEM accumulator; the S of the next sub-tile is issued before the P V of
//    this one, so the tensor core computes while the softmax runs;
//  * warps 0-3 and 4-7: one softmax warpgroup per M tile, a thread per row
//    (TMEM lane): reads S, masks (causal on the diagonal block, the sequence
//    end), online softmax in the exp2 domain with a lazily moved reference
//    maximum (O and l are rescaled in TMEM only when the row maximum grows by
//    more than 2^8), writes P as bf16 into shared memory in the MMA's operand
//    layout; at the end reads O, divides by l and stores the row;
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
constexpr int kSub = 64;            // key tokens per sub-tile
constexpr int kTmemCols = 512;
constexpr int kAttnSmemLimit = 232448;
constexpr int kMaxAttnStages = 8;
constexpr float kLog2eA = 1.44269504088896340736f;
constexpr float kLn2A = 0.69314718055994530942f;
constexpr float kRescaleLog2 = 8.0f;  // move the reference maximum only past a 2^8 growth
constexpr int kListCap = 384;         // kept lists up to this length are staged in shared memory

template <int D>
struct AttnCfg {
    static constexpr int kBoxes = D / 64;               // 128-byte column boxes of a row
    static constexpr int kQTile = kBoxes * 128 * 128;   // one M tile of Q
    static constexpr int kPTile = 128 * 128;            // one M tile of P (64 tokens)
    static constexpr int kKV = kBoxes * kSub * 128;     // K (or V) of one sub-tile
    static constexpr int kStage = 2 * kKV;
    static constexpr int kFixed = 2 * kQTile + 2 * kPTile;
    static constexpr int kBarBytes = 256 + kListCap * 4;
    static constexpr int kStages0 = (kAttnSmemLimit - 1024 - kBarBytes - kFixed) / kStage;
    static constexpr int kStages = kStages0 > kMaxAttnStages ? kMaxAttnStages : kStages0;
    static constexpr int kSmem = 1024 + kFixed + kStages * kStage + kBarBytes;
    static constexpr int kOCol = 0;                     // per tile: O at +0, S buffers at +D, +D+64
    static_assert(kStages >= 2, "too little shared memory for the K/V ring");
    static_assert(D + 2 * kSub <= kTmemCols / 2, "TMEM columns of one tile");
};

// The kept (b, kvh, i) list walked as 64-token sub-tiles: entries outside
// [0, i] are skipped, and so is a second half that starts at or past L.
struct SubIter {
    const int32_t* list;
    int nsel, i, L, blk, halves;
    int x, hh, j;
    __device__ void seek() {
        while (x < nsel) {
            j = list[x];
            if (j >= 0 && j <= i && j * blk + kSub * hh < L) return;
            ++x;
            hh = 0;
        }
    }
    __device__ void start() {
        x = 0;
        hh = 0;
        seek();
    }
    __device__ bool done() const { return x >= nsel; }
    __device__ int tok0() const { return j * blk + kSub * hh; }
    __device__ void next() {
        if (++hh == halves) {
            hh = 0;
            ++x;
        }
        seek();
    }
};

struct AttnBars {
    uint32_t q_full, kv_full, kv_empty, s_ready, s_free, p_ready, pv_done, drain;
    // kv_full / kv_empty: + 8 * stage; s_ready / s_free: + 8 * (2 * tile + buffer); p_ready / pv_done: + 8 * tile
};

// 2^x on the special-function unit (flush-to-zero; 2^-inf = 0).
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
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

    // ---- shared memory: Q tiles, P tiles, K/V stages, barriers
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char* gbase = smem_raw + (base - raw);
    const uint32_t sQ = base, sP = base + 2 * C::kQTile, sKV = sP + 2 * C::kPTile;
    const uint32_t sBar = sKV + C::kStages * C::kStage;
    unsigned char* gBar = gbase + (sBar - base);
    AttnBars bars;
    bars.q_full = sBar;
    bars.kv_full = sBar + 8;
    bars.kv_empty = bars.kv_full + 8 * C::kStages;
    bars.s_ready = bars.kv_empty + 8 * C::kStages;
    bars.s_free = bars.s_ready + 8 * 4;
    bars.p_ready = bars.s_free + 8 * 4;
    bars.pv_done = bars.p_ready + 8 * 2;
    bars.drain = bars.pv_done + 8 * 2;
    const uint32_t bar_end = bars.drain + 8;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gBar + (bar_end - sBar));
    int* abort_flag = reinterpret_cast<int*>(gBar + (bar_end - sBar) + 4);
    int32_t* list_s = reinterpret_cast<int32_t*>(gBar + 256);

    if (tid == 0) {
        mbar_init(bars.q_full, 1);
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(bars.kv_full + 8 * s, 1);
            mbar_init(bars.kv_empty + 8 * s, 1);
        }
        for (int x = 0; x < 4; ++x) {
            mbar_init(bars.s_ready + 8 * x, 1);
            mbar_init(bars.s_free + 8 * x, 4);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(bars.p_ready + 8 * t, 4);
            mbar_init(bars.pv_done + 8 * t, 1);
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

    SubIter it0;
    it0.list = list;
    it0.nsel = nsel;
    it0.i = i;
    it0.L = L;
    it0.blk = BLK;
    it0.halves = BLK / kSub;
    it0.start();
    const bool any = !it0.done();

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
            SubIter it = it0;
            int n = 0;
            for (; !it.done(); it.next(), ++n) {
                const int st = n % C::kStages;
                if (n >= C::kStages && !mbar_wait(bars.kv_empty + 8 * st, (uint32_t)((n / C::kStages - 1) & 1))) {
                    fail();
                    break;
                }
                if (abort_set(abort_flag)) break;
                const uint32_t stage = sKV + st * C::kStage;
                const uint32_t bar = bars.kv_full + 8 * st;
                mbar_arrive_expect_tx(bar, (uint32_t)C::kStage);
                const int y = row * Lmax + it.tok0();
                for (int c = 0; c < C::kBoxes; ++c) {
                    tma_load_2d(stage + c * kSub * 128, &tmK, bar, c * 64, y, keep);
                    tma_load_2d(stage + C::kKV + c * kSub * 128, &tmV, bar, c * 64, y, keep);
                }
            }
            // leave only after the copies issued have landed
            const int issued = n;
            for (int m = max(0, issued - C::kStages); m < issued; ++m)
                (void)mbar_wait(bars.kv_full + 8 * (m % C::kStages), (uint32_t)((m / C::kStages) & 1));
            (void)mbar_wait(bars.q_full, 0u);
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ---------------------------------------------------------------- MMA issue
        if (lane == 0 && any) {
            constexpr uint32_t kIdS = tc::idesc_bf16_f32(128, kSub, false);
            constexpr uint32_t kIdO = tc::idesc_bf16_f32(128, D, true);
            bool ok = mbar_wait(bars.q_full, 0u);
            const uint64_t dq0 = tc::smem_desc_sw128(sQ, 16, 1024);
            const uint64_t dq1 = tc::smem_desc_sw128(sQ + C::kQTile, 16, 1024);
            const uint64_t dp0 = tc::smem_desc_sw128(sP, 16, 1024);
            const uint64_t dp1 = tc::smem_desc_sw128(sP + C::kPTile, 16, 1024);
            // S_t(n) = Q_t K(n)^T into buffer n % 2 of tile t
            auto issue_s = [&](int n) -> bool {
                const int st = n % C::kStages;
                if (!mbar_wait(bars.kv_full + 8 * st, (uint32_t)((n / C::kStages) & 1))) return false;
                const uint64_t dk = tc::smem_desc_sw128(sKV + st * C::kStage, 16, 1024);
                for (int t = 0; t < n_tiles; ++t) {
                    const int buf = n & 1;
                    if (n >= 2 && !mbar_wait(bars.s_free + 8 * (2 * t + buf), (uint32_t)(((n - 2) >> 1) & 1)))
                        return false;
                    tc::fence_after_sync();
                    const uint32_t d_tmem = tmem + (uint32_t)(t * (kTmemCols / 2) + D + buf * kSub);
                    const uint64_t dq = t == 0 ? dq0 : dq1;
                    // k-th 16-column step: box k / 4, 32 bytes * (k % 4) into the swizzled row
#pragma unroll
                    for (int k = 0; k < D / 16; ++k)
                        tc::mma_bf16_ss(d_tmem, dq + (uint64_t)((k >> 2) * (128 * 128 / 16) + (k & 3) * 2),
                                        dk + (uint64_t)((k >> 2) * (kSub * 128 / 16) + (k & 3) * 2), kIdS, k > 0);
                    tc::commit(bars.s_ready + 8 * (2 * t + buf));
                }
                return true;
            };
            SubIter it = it0;
            int n = 0;
            if (ok) ok = issue_s(0);
            while (ok && !it.done()) {
                SubIter nx = it;
                nx.next();
                if (!nx.done()) {
                    ok = issue_s(n + 1);
                    if (!ok) break;
                }
                const uint64_t dv = tc::smem_desc_sw128(sKV + (n % C::kStages) * C::kStage + C::kKV, kSub * 128, 1024);
                for (int t = 0; t < n_tiles; ++t) {
                    if (!mbar_wait(bars.p_ready + 8 * t, (uint32_t)(n & 1))) {
                        ok = false;
                        break;
                    }
                    tc::fence_after_sync();
                    const uint32_t o_tmem = tmem + (uint32_t)(t * (kTmemCols / 2));
                    const uint64_t dp = t == 0 ? dp0 : dp1;
                    // k-th 16-token step: 32 bytes into each P row, 16 V rows further
#pragma unroll
                    for (int k = 0; k < kSub / 16; ++k)
                        tc::mma_bf16_ss(o_tmem, dp + (uint64_t)(k * 2), dv + (uint64_t)(k * (16 * 128 / 16)), kIdO,
                                        n > 0 || k > 0);
                    tc::commit(bars.pv_done + 8 * t);
                }
                if (!ok) break;
                tc::commit(bars.kv_empty + 8 * (n % C::kStages));  // S(n) and P V(n) read the stage
                if (abort_set(abort_flag)) {
                    ok = false;
                    break;
                }
                it = nx;
                ++n;
            }
            if (!ok) fail();
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
        const uint32_t p_row = sP + t * C::kPTile + r * 128;
        float m_ref = -INFINITY, l = 0.f;
        bool ok = true;
        SubIter it = it0;
        int n = 0;
        for (; !it.done(); it.next(), ++n) {
            const int buf = n & 1;
            bool w = mbar_wait(bars.s_ready + 8 * (2 * t + buf), (uint32_t)((n >> 1) & 1));
            if (__any_sync(0xffffffffu, !w || abort_set(abort_flag))) {  // one decision for the warp
                ok = false;
                break;
            }
            tc::fence_after_sync();
            uint32_t s[2][32];
            tc::ld_32x32b_x32(t_tmem + (uint32_t)(D + buf * kSub), s[0]);
            tc::ld_32x32b_x32(t_tmem + (uint32_t)(D + buf * kSub + 32), s[1]);
            tc::wait_ld();
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(bars.s_free + 8 * (2 * t + buf));
            // mask (only the diagonal and the sequence end), then the row maximum of the raw scores
            const int lim = lim_tok - it.tok0();   // columns 0 .. lim are visible
            if (!__all_sync(0xffffffffu, lim >= kSub - 1)) {
#pragma unroll
                for (int c = 0; c < kSub; ++c)
                    if (c > lim) s[c >> 5][c & 31] = __float_as_uint(-INFINITY);
            }
            float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int c = 0; c < kSub; ++c) m4[c & 3] = fmaxf(m4[c & 3], __uint_as_float(s[c >> 5][c & 31]));
            const float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * scale_log2;  // scale > 0
            float alpha = 1.f;
            if (mx > m_ref + kRescaleLog2 || (m_ref == -INFINITY && mx > -INFINITY)) {
                alpha = m_ref == -INFINITY ? 0.f : ex2(m_ref - mx);
                m_ref = mx;
                l *= alpha;
            }
            const float neg_m = m_ref == -INFINITY ? 0.f : -m_ref;
            uint32_t pk[kSub / 2];
            float sum2[2] = {0.f, 0.f};
#pragma unroll
            for (int c = 0; c < kSub; c += 2) {
                const float p0 = ex2(fmaf(__uint_as_float(s[c >> 5][c & 31]), scale_log2, neg_m));
                const float p1 = ex2(fmaf(__uint_as_float(s[(c + 1) >> 5][(c + 1) & 31]), scale_log2, neg_m));
                sum2[(c >> 1) & 1] += p0 + p1;
                pk[c / 2] = pack_bf16x2(p0, p1);
            }
            l += sum2[0] + sum2[1];
            // P and O are free once the previous P V has completed
            if (n > 0) {
                w = mbar_wait(bars.pv_done + 8 * t, (uint32_t)((n - 1) & 1));
                if (__any_sync(0xffffffffu, !w)) {
                    ok = false;
                    break;
                }
                tc::fence_after_sync();
            }
#pragma unroll
            for (int ch = 0; ch < 8; ++ch)
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(p_row + ((ch ^ (r & 7)) << 4)),
                             "r"(pk[4 * ch]), "r"(pk[4 * ch + 1]), "r"(pk[4 * ch + 2]), "r"(pk[4 * ch + 3])
                             : "memory");
            if (n > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
                for (int c0 = 0; c0 < D; c0 += 32) {
                    uint32_t o[32];
                    tc::ld_32x32b_x32(t_tmem + (uint32_t)(C::kOCol + c0), o);
                    tc::wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                    tc::st_32x32b_x32(t_tmem + (uint32_t)(C::kOCol + c0), o);
                }
                tc::wait_st();
            }
            // the sequence end inside this sub-tile: zero the V rows past it (they may hold anything)
            if (t == 0 && it.tok0() + kSub > L) {
                const int v0 = L - it.tok0();
                const uint32_t sv = sKV + (n % C::kStages) * C::kStage + C::kKV;
                for (int x = (warp & 3) * 32 + lane; x < (kSub - v0) * C::kBoxes * 8; x += 128) {
                    const int rr = v0 + x / (C::kBoxes * 8), rem = x % (C::kBoxes * 8);
                    const uint32_t a = sv + (rem >> 3) * (kSub * 128) + rr * 128 + (rem & 7) * 16;
                    asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(0u) : "memory");
                }
            }
            fence_proxy_async_smem();
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(bars.p_ready + 8 * t);
        }
        // ---- epilogue: O / l
        if (ok && n > 0) {
            const bool w = mbar_wait(bars.pv_done + 8 * t, (uint32_t)((n - 1) & 1));
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
            tc::ld_32x32b_x32(t_tmem + (uint32_t)(C::kOCol + c0), o);
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
