// combine.cu -- log-sum-exp merge of the split-KV partial outputs.
//
// Each (b, h) has S slots of (o_s, lse_s) over disjoint token sets; the
// softmax over their union is
//   M = max_s lse_s,  w_s = exp(lse_s - M),
//   out = sum_s w_s o_s / sum_s w_s,  lse = M + log sum_s w_s.
// Slots with lse = -inf hold no token and are skipped (their o is never
// read). One warp per (b, h): lanes scan the S lse values, then walk the live
// slots found by a ballot, each lane owning D/32 contiguous output columns.
#include <cmath>

#include "seer_device.cuh"
#include "seer_launch.h"

namespace seer {
namespace {

constexpr int kWarpsPerCta = 4;

template <int D>
__global__ void __launch_bounds__(kWarpsPerCta * 32)
    combine_kernel(const float* __restrict__ o_part, const float* __restrict__ lse_part, int S, int BH,
                   __nv_bfloat16* __restrict__ out, float* __restrict__ lse_out) {
    after_prior_grid();
    constexpr int kVec = D / 32;
    const int lane = threadIdx.x & 31;
    const int bh = blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
    if (bh >= BH) return;
    const float* l = lse_part + (size_t)bh * S;
    float M = -INFINITY;
    for (int s = lane; s < S; s += 32) M = fmaxf(M, l[s]);
    M = warp_max(M);
    __nv_bfloat16* dst = out + (size_t)bh * D + lane * kVec;
    if (M == -INFINITY) {
#pragma unroll
        for (int u = 0; u < kVec; ++u) dst[u] = __float2bfloat16(0.f);
        if (lse_out && lane == 0) lse_out[bh] = -INFINITY;
        return;
    }
    float acc[kVec];
#pragma unroll
    for (int u = 0; u < kVec; ++u) acc[u] = 0.f;
    float wsum = 0.f;
    const float* o = o_part + (size_t)bh * S * D + lane * kVec;
    for (int base = 0; base < S; base += 32) {
        const int s = base + lane;
        const float ls = s < S ? l[s] : -INFINITY;
        const float w = (ls == -INFINITY) ? 0.f : expf(ls - M);
        unsigned live = __ballot_sync(0xffffffffu, ls != -INFINITY);
        while (live) {
            const int k = __ffs(live) - 1;
            live &= live - 1;
            const float wk = __shfl_sync(0xffffffffu, w, k);
            const float* src = o + (size_t)(base + k) * D;
            if constexpr (kVec == 4) {
                const float4 v = *reinterpret_cast<const float4*>(src);
                acc[0] += wk * v.x;
                acc[1] += wk * v.y;
                acc[2] += wk * v.z;
                acc[3] += wk * v.w;
            } else {
                const float2 v = *reinterpret_cast<const float2*>(src);
                acc[0] += wk * v.x;
                acc[1] += wk * v.y;
            }
            wsum += wk;
        }
    }
    const float inv = 1.f / wsum;
    if constexpr (kVec == 4) {
        __nv_bfloat162 lo = __floats2bfloat162_rn(acc[0] * inv, acc[1] * inv);
        __nv_bfloat162 hi = __floats2bfloat162_rn(acc[2] * inv, acc[3] * inv);
        uint2 pk;
        pk.x = *reinterpret_cast<uint32_t*>(&lo);
        pk.y = *reinterpret_cast<uint32_t*>(&hi);
        *reinterpret_cast<uint2*>(dst) = pk;
    } else {
        *reinterpret_cast<__nv_bfloat162*>(dst) = __floats2bfloat162_rn(acc[0] * inv, acc[1] * inv);
    }
    if (lse_out && lane == 0) lse_out[bh] = M + logf(wsum);
}

}  // namespace

cudaError_t launch_combine(const Shape& s, const float* o_part, const float* lse_part, int num_splits, void* out,
                           float* lse_out, cudaStream_t stream) {
    const int BH = s.B * s.Hq;
    const int grid = (BH + kWarpsPerCta - 1) / kWarpsPerCta;
    auto* o = static_cast<__nv_bfloat16*>(out);
    if (s.D == 128)
        return launch_after_prior(combine_kernel<128>, dim3(grid), dim3(kWarpsPerCta * 32), 0, stream, nullptr,
                                  o_part, lse_part, num_splits, BH, o, lse_out);
    return launch_after_prior(combine_kernel<64>, dim3(grid), dim3(kWarpsPerCta * 32), 0, stream, nullptr, o_part,
                              lse_part, num_splits, BH, o, lse_out);
}

}  // namespace seer
