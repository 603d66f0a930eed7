// seer_device.cuh -- small device helpers for the sm_100a kernels: shared
// memory addresses, mbarriers with bounded waits, TMA / bulk copies,
// ldmatrix and mma.sync wrappers, warp reductions.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

namespace seer {

// A wait on an mbarrier gives up after this long. Every wait in these kernels
// normally completes within microseconds; the limit only turns a logic error
// into a reported failure instead of a hung GPU.
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---------------------------------------------------------------- mbarrier

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    return done != 0;
}

// Wait for the phase of `parity` to complete; false once `limit_ns` has passed.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 32; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (global_timer_ns() - t0 > limit_ns) return false;
    }
}

// Order this thread's generic-proxy shared-memory writes before later
// async-proxy (TMA) accesses of the same memory.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------- TMA / bulk copies

__device__ __forceinline__ void prefetch_tensor_map(const void* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// 2-D tiled TMA load into this CTA's shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* map, uint32_t bar, int x, int y,
                                            uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(dst),
        "l"(map), "r"(bar), "r"(x), "r"(y), "l"(policy)
        : "memory");
}

// Plain (untiled) bulk copy global -> shared; 16-byte aligned, size % 16 == 0.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// ---------------------------------------------------------------- tensor-core fragments

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                            uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                                  uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

// D = A(16x16, row) * B(16x8, col) + D, bf16 in, fp32 accumulate.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D = A(16x8, row) * B(8x8, col) + D, bf16 in, fp32 accumulate.
__device__ __forceinline__ void mma_bf16_1688(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5}, {%6}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(b0));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// ---------------------------------------------------------------- misc

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// out[e] = W[e, :] . v for the rows e = first, first + stride, ... < end, one
// warp per row with 8 rows in flight: each lane holds D/32 entries of v
// (vd) and reads the matching 16- or 8-byte piece of each W row (coalesced
// across the warp). Lane 0 of the warp returns the dot through `sink`.
// One lane's piece of a W-row . v dot (4 or 2 columns); every matvec of the
// library goes through these, so equal inputs give equal bits.
// Read-only vector loads that stay where they are written (volatile asm keeps
// them ahead of the barriers that follow), for loads issued early on purpose.
__device__ __forceinline__ void load_early(float4& x, const float* p) {
    asm volatile("ld.global.nc.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(x.x), "=f"(x.y), "=f"(x.z), "=f"(x.w)
                 : "l"(p));
}
__device__ __forceinline__ void load_early(float2& x, const float* p) {
    asm volatile("ld.global.nc.v2.f32 {%0, %1}, [%2];" : "=f"(x.x), "=f"(x.y) : "l"(p));
}
__device__ __forceinline__ int load_early(const int32_t* p) {
    int x;
    asm volatile("ld.global.nc.s32 %0, [%1];" : "=r"(x) : "l"(p));
    return x;
}

__device__ __forceinline__ float piece_dot(const float4& w, const float* v) {
    return w.x * v[0] + w.y * v[1] + w.z * v[2] + w.w * v[3];
}
__device__ __forceinline__ float piece_dot(const float2& w, const float* v) { return w.x * v[0] + w.y * v[1]; }

template <int D, typename Sink>
__device__ __forceinline__ void warp_matvec_rows(const float* __restrict__ W, const float (&vd)[D / 32], int first,
                                                 int end, int stride, Sink sink) {
    constexpr int kVec = D / 32;
    const int lane = threadIdx.x & 31;
    for (int e0 = first; e0 < end; e0 += 8 * stride) {
        float d[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int e = e0 + u * stride;
            d[u] = 0.f;
            if (e < end) {
                const float* we = W + (size_t)e * D + lane * kVec;
                if constexpr (kVec == 4) d[u] = piece_dot(*reinterpret_cast<const float4*>(we), vd);
                else d[u] = piece_dot(*reinterpret_cast<const float2*>(we), vd);
            }
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            float x = d[u];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
            const int e = e0 + u * stride;
            if (lane == 0 && e < end) sink(e, x);
        }
    }
}

// atomicAdd with acquire-release semantics at GPU scope: publishes every write
// this thread has observed (e.g. its CTA's writes before a __syncthreads) and
// sees every write published by earlier adds to the same counter.
__device__ __forceinline__ unsigned int atomic_add_acq_rel(unsigned int* p, unsigned int v) {
    unsigned int old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

// Named barrier over `threads` threads (a multiple of 32), id 1..15.
__device__ __forceinline__ void named_barrier_sync(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

__device__ __forceinline__ int clamp_len(int len, int lmax) { return len < 0 ? 0 : (len > lmax ? lmax : len); }

// Kernels of the separate calls are launched so that they may start while the
// stream's previous kernel finishes (programmatic dependent launch). Each one
// first waits for that kernel's completion and the visibility of its writes,
// then lets the stream's next kernel launch: nothing is read early.
__device__ __forceinline__ void after_prior_grid() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Host side: launch `kernel` with that permission (and the given extra attribute, if any).
template <typename... KArgs, typename... Args>
cudaError_t launch_after_prior(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                               const cudaLaunchAttribute* extra, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    if (extra) attr[1] = *extra;
    cfg.attrs = attr;
    cfg.numAttrs = extra ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

}  // namespace seer
