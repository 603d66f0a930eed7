// block_mass.cu -- block-level ground truth of one decode query.
//
// "SeerAttention: Learning Intrinsic Sparse Attention in Your LLMs"
// (abstract) trains its gate against a block-level ground truth extracted by
// a customised attention kernel; "SeerAttention-R" (abstract) keeps that
// self-distilled gate for decoding. For a decode query this target is the
// share of each query head's dense softmax that falls in each KV block:
//
//   z_t     = scale * q_h . K[b, kvh, t]            t < L_b
//   mass[j] = sum_{t in block j} exp(z_t) / sum_t exp(z_t)      (0 for j >= NB_b)
//   lse     = log sum_t exp(z_t)
//
// Pass 1 (block_lse_kernel): one warp per KV block. The warp copies the
// block's K tile, 64 tokens at a time, into its own shared-memory ring with
// 16-byte cp.async (rows padded by 16 bytes so that ldmatrix reads are
// conflict-free; three stages, two tiles in flight), computes Q K^T on the tensor
// cores (mma.sync bf16 -> fp32, the G query heads as the M side, tokens as
// N), and reduces each head's logits over the block inside the warp: the
// block's log-mass m + log(sum exp(z - m)) goes to `mass` as scratch. No CTA
// barrier anywhere: the pass streams K once, HBM-bound.
// Pass 2 (block_mass_finalize_kernel): one warp per (b, query head) turns the
// row's block log-masses into lse and mass in place.
#include <cuda_bf16.h>

#include "seer_device.cuh"
#include "seer_launch.h"

namespace seer {
namespace {

constexpr float kLog2eF = 1.44269504088896340736f;
constexpr float kLn2F = 0.69314718055994530942f;

template <int D, int BLK>
struct MassCfg {
    static constexpr int kSub = 64;                      // tokens per staged tile (a block is BLK / 64 tiles)
    static constexpr int kNSub = BLK / kSub;
    static constexpr int kWarps = 4;
    static constexpr int kRowBytes = D * 2 + 16;         // padded tile row: conflict-free ldmatrix
    static constexpr int kBufBytes = kSub * kRowBytes;   // one staged tile
    static constexpr int kStages = 3;                    // per warp: two tiles in flight, one computed
    static constexpr int kSmem = kWarps * kStages * kBufBytes;
    static constexpr int kBlocksPerWarp = 16 / kNSub;    // 16 tiles per warp
    static constexpr int kBlocksPerCta = kWarps * kBlocksPerWarp;
    static constexpr int kTiles = kBlocksPerWarp * kNSub;
    static constexpr int kKSteps = D / 16;
    static constexpr int kNT8 = kSub / 8;                // n8 token tiles per staged tile
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Copies the valid rows of the 64 tokens starting at token t0 into buffer `dst` (one warp).
template <int D, int BLK>
__device__ __forceinline__ void load_tile(uint32_t dst, const __nv_bfloat16* krow, int t0, int L, int lane) {
    using C = MassCfg<D, BLK>;
    const int nrows = min(C::kSub, L - t0);
    const __nv_bfloat16* src = krow + (size_t)t0 * D;
    constexpr int kPerRow = D * 2 / 16;
    for (int c = lane; c < nrows * kPerRow; c += 32) {
        const int r = c / kPerRow, q = c - r * kPerRow;
        cp_async16(dst + r * C::kRowBytes + q * 16, src + (size_t)r * D + q * 8);
    }
}

template <int D, int BLK>
__global__ void __launch_bounds__(MassCfg<D, BLK>::kWarps * 32)
    block_lse_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k_cache,
                     const int32_t* __restrict__ seq_lens, int Hq, int Hkv, int Lmax, int NBmax, float scale_log2,
                     float* __restrict__ blse) {
    using C = MassCfg<D, BLK>;
    extern __shared__ __align__(16) unsigned char smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, tig = lane & 3;
    const int row = blockIdx.y;
    const int b = row / Hkv, kvh = row - b * Hkv;
    const int G = Hq / Hkv;
    const int L = clamp_len(seq_lens[b], Lmax);
    const int NB = (L + BLK - 1) / BLK;
    const int j0 = blockIdx.x * C::kBlocksPerCta + warp;  // this warp: blocks j0, j0 + kWarps, ...
    if (j0 >= NB) return;
    const __nv_bfloat16* krow = k_cache + (size_t)row * Lmax * D;
    const uint32_t buf0 = smem_addr(smem) + warp * C::kStages * C::kBufBytes;
    // the warp's staged tile u is half u % kNSub of its block u / kNSub
    auto tile_t0 = [&](int u) { return (j0 + (u / C::kNSub) * C::kWarps) * BLK + (u % C::kNSub) * C::kSub; };
    const int ntiles = min(C::kTiles, ((NB - 1 - j0) / C::kWarps + 1) * C::kNSub);

    // query fragments of the group's heads (rows g < G of the M = 16 side)
    uint32_t qa[C::kKSteps][2];
    const __nv_bfloat16* qh = q + ((size_t)b * Hq + (size_t)kvh * G + (g < G ? g : 0)) * D;
#pragma unroll
    for (int kk = 0; kk < C::kKSteps; ++kk) {
        qa[kk][0] = g < G ? *reinterpret_cast<const uint32_t*>(qh + kk * 16 + 2 * tig) : 0u;
        qa[kk][1] = g < G ? *reinterpret_cast<const uint32_t*>(qh + kk * 16 + 8 + 2 * tig) : 0u;
    }

    // stage s of the warp's ring holds its tiles u = s, s + 3, ...; one commit group per tile
    for (int u = 0; u < C::kStages - 1; ++u) {
        if (u < ntiles) load_tile<D, BLK>(buf0 + u * C::kBufBytes, krow, tile_t0(u), L, lane);
        cp_async_commit();
    }
    float M = -INFINITY, S = 0.f;  // the current block's running max and sum (log2 domain)
    for (int u = 0; u < ntiles; ++u) {
        const int ua = u + C::kStages - 1;  // tile issued now
        if (ua < ntiles) load_tile<D, BLK>(buf0 + (ua % C::kStages) * C::kBufBytes, krow, tile_t0(ua), L, lane);
        cp_async_commit();  // possibly empty: keeps one group per tile
        cp_async_wait<C::kStages - 1>();
        __syncwarp();
        const uint32_t cur = buf0 + (u % C::kStages) * C::kBufBytes;
        const int valid = min(C::kSub, L - tile_t0(u));  // <= 0: the empty half of a partial block
        float x[C::kNT8][2];
#pragma unroll
        for (int nt = 0; nt < C::kNT8; ++nt) {
            float s[4] = {0.f, 0.f, 0.f, 0.f};
            const int tok = nt * 8 + (lane & 7);
            const int mi = lane >> 3;
            if (nt * 8 < valid) {  // warp-uniform: tiles past the length hold no copied rows
#pragma unroll
                for (int kk2 = 0; kk2 < C::kKSteps / 2; ++kk2) {
                    uint32_t r0, r1, r2, r3;
                    ldmatrix_x4(cur + tok * C::kRowBytes + ((2 * kk2 + (mi >> 1)) * 16 + (mi & 1) * 8) * 2, r0, r1, r2,
                                r3);
                    mma_bf16_16816(s, qa[2 * kk2][0], 0u, qa[2 * kk2][1], 0u, r0, r1);
                    mma_bf16_16816(s, qa[2 * kk2 + 1][0], 0u, qa[2 * kk2 + 1][1], 0u, r2, r3);
                }
            }
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int t = nt * 8 + 2 * tig + e;
                x[nt][e] = t < valid ? s[e] * scale_log2 : -INFINITY;
            }
        }
        float m = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < C::kNT8; ++nt) m = fmaxf(m, fmaxf(x[nt][0], x[nt][1]));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
        const float Mn = fmaxf(M, m);
        if (Mn != -INFINITY) {
            float sum = 0.f;
#pragma unroll
            for (int nt = 0; nt < C::kNT8; ++nt) sum += exp2f(x[nt][0] - Mn) + exp2f(x[nt][1] - Mn);
            sum += __shfl_xor_sync(0xffffffffu, sum, 1);
            sum += __shfl_xor_sync(0xffffffffu, sum, 2);
            S = S * exp2f(M - Mn) + sum;  // M = -inf: S is 0 and the factor is 0
            M = Mn;
        }
        if (u % C::kNSub == C::kNSub - 1) {  // the block's last tile: write its log-mass
            const int j = j0 + (u / C::kNSub) * C::kWarps;
            if (tig == 0 && g < G) blse[((size_t)b * Hq + (size_t)kvh * G + g) * NBmax + j] = (M + log2f(S)) * kLn2F;
            M = -INFINITY;
            S = 0.f;
        }
        __syncwarp();  // the stage is refilled on the next step
    }
    cp_async_wait<0>();
}

// Pass 2: one warp per (b, query head). Reads the row's block log-masses,
// forms lse = log sum_j exp(blse_j) and rewrites the row as mass_j =
// exp(blse_j - lse) (0 for j >= NB_b, and lse = -inf for an empty row).
__global__ void __launch_bounds__(256)
    block_mass_finalize_kernel(const int32_t* __restrict__ seq_lens, int B, int Hq, int Lmax, int blk, int NBmax,
                               float* __restrict__ mass, float* __restrict__ lse_out) {
    const int w = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (w >= B * Hq) return;
    const int b = w / Hq;
    const int NB = (clamp_len(seq_lens[b], Lmax) + blk - 1) / blk;
    float* r = mass + (size_t)w * NBmax;
    float M = -INFINITY;
    for (int j = lane; j < NB; j += 32) M = fmaxf(M, r[j]);
    M = warp_max(M);
    float s = 0.f;
    if (M != -INFINITY)
        for (int j = lane; j < NB; j += 32) s += expf(r[j] - M);
    s = warp_sum(s);
    const float lse = M == -INFINITY ? -INFINITY : M + logf(s);
    for (int j = lane; j < NBmax; j += 32) r[j] = j < NB ? expf(r[j] - lse) : 0.f;
    if (lane == 0 && lse_out) lse_out[w] = lse;
}

template <int D, int BLK>
cudaError_t mass_impl(const Shape& s, const void* q, const void* k_cache, const int32_t* seq_lens, float sm_scale,
                      float* mass, float* lse_out, cudaStream_t stream) {
    using C = MassCfg<D, BLK>;
    static bool attr_done = false;  // once per template instance (benign race)
    if (!attr_done) {
        cudaError_t e = cudaFuncSetAttribute(block_lse_kernel<D, BLK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             C::kSmem);
        if (e != cudaSuccess) return e;
        attr_done = true;
    }
    const dim3 grid((s.NBmax + C::kBlocksPerCta - 1) / C::kBlocksPerCta, s.B * s.Hkv);
    block_lse_kernel<D, BLK><<<grid, C::kWarps * 32, C::kSmem, stream>>>(
        static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k_cache), seq_lens, s.Hq, s.Hkv,
        s.Lmax, s.NBmax, sm_scale * kLog2eF, mass);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    block_mass_finalize_kernel<<<(s.B * s.Hq + 7) / 8, 256, 0, stream>>>(seq_lens, s.B, s.Hq, s.Lmax, s.blk,
                                                                           s.NBmax, mass, lse_out);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_block_mass(const Shape& s, const void* q, const void* k_cache, const int32_t* seq_lens,
                              float sm_scale, float* mass, float* lse_out, cudaStream_t stream) {
    if (s.D == 128 && s.blk == 64) return mass_impl<128, 64>(s, q, k_cache, seq_lens, sm_scale, mass, lse_out, stream);
    if (s.D == 128 && s.blk == 128) return mass_impl<128, 128>(s, q, k_cache, seq_lens, sm_scale, mass, lse_out, stream);
    if (s.D == 64 && s.blk == 64) return mass_impl<64, 64>(s, q, k_cache, seq_lens, sm_scale, mass, lse_out, stream);
    if (s.D == 64 && s.blk == 128) return mass_impl<64, 128>(s, q, k_cache, seq_lens, sm_scale, mass, lse_out, stream);
    return cudaErrorInvalidValue;
}

}  // namespace seer
