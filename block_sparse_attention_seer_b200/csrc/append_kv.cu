// append_kv.cu -- write the decode step's new token into the KV caches.
//
// "SeerAttention-R: Sparse Attention Adaptation for Long Reasoning"
// (abstract) decodes auto-regressively: each step appends one token, whose K
// and V rows then take part in that same step (the open last block is always
// kept, and its pooled key is refreshed from the cache). This kernel puts the
// token's rows at position L_b - 1 of every (b, kv head) row of the caches, so
// a caller ships only q and the new K/V per step instead of writing strided
// cache slices itself.
//
// One warp per (b, kv head): D bf16 values of K and of V, 16-byte stores.
#include <cuda_bf16.h>

#include "seer_device.cuh"
#include "seer_launch.h"

namespace seer {
namespace {

constexpr int kWarpsPerCta = 8;

template <int D>
__global__ void __launch_bounds__(kWarpsPerCta * 32)
    append_kv_kernel(const __nv_bfloat16* __restrict__ k_new, const __nv_bfloat16* __restrict__ v_new,
                     const int32_t* __restrict__ seq_lens, int rows, int Hkv, int Lmax,
                     __nv_bfloat16* __restrict__ k_cache, __nv_bfloat16* __restrict__ v_cache) {
    constexpr int kVec = D * 2 / 16;  // 16-byte pieces of one row (8 or 16)
    const int row = blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const int L = clamp_len(seq_lens[row / Hkv], Lmax);
    if (L == 0) return;  // no token to place
    const size_t dst = ((size_t)row * Lmax + (L - 1)) * D;
    const size_t src = (size_t)row * D;
    if (lane < kVec) {
        reinterpret_cast<uint4*>(k_cache + dst)[lane] = reinterpret_cast<const uint4*>(k_new + src)[lane];
    } else if (lane < 2 * kVec) {
        reinterpret_cast<uint4*>(v_cache + dst)[lane - kVec] =
            reinterpret_cast<const uint4*>(v_new + src)[lane - kVec];
    }
}

}  // namespace

cudaError_t launch_append_kv(const Shape& s, const void* k_new, const void* v_new, const int32_t* seq_lens,
                             void* k_cache, void* v_cache, cudaStream_t stream) {
    const int rows = s.B * s.Hkv;
    const dim3 grid((rows + kWarpsPerCta - 1) / kWarpsPerCta), block(kWarpsPerCta * 32);
    auto kn = static_cast<const __nv_bfloat16*>(k_new);
    auto vn = static_cast<const __nv_bfloat16*>(v_new);
    auto kc = static_cast<__nv_bfloat16*>(k_cache);
    auto vc = static_cast<__nv_bfloat16*>(v_cache);
    if (s.D == 128) append_kv_kernel<128><<<grid, block, 0, stream>>>(kn, vn, seq_lens, rows, s.Hkv, s.Lmax, kc, vc);
    else if (s.D == 64) append_kv_kernel<64><<<grid, block, 0, stream>>>(kn, vn, seq_lens, rows, s.Hkv, s.Lmax, kc, vc);
    else return cudaErrorInvalidValue;
    return cudaGetLastError();
}

}  // namespace seer
