// prefill.cu -- block-sparse attention over a causal prompt.
//
// "SeerAttention: Learning Intrinsic Sparse Attention in Your LLMs"
// (abstract) pools Q and K along the sequence, passes them through learnable
// linear layers, multiplies the results into block-level gating scores, and
// runs a block-sparse FlashAttention over the kept blocks. With the decode
// gate's readings (mean pooling over valid tokens, one bias-free map per KV
// head, mean over the group's heads, 1/sqrt(dg)) this is, for a prompt of L_b
// tokens with query / key blocks of `blk` tokens:
//
//   gate:   s[b,kvh,i,j] = (W_q qbar_i) . kpool[b,kvh,j] / sqrt(dg),  j <= i,
//           qbar_i = the mean of the group's queries over query block i
//   select: block i itself plus the top min(k, i+1) - 1 of blocks 0 .. i-1
//           (the decode rule on a sequence of i + 1 blocks)
//   attend: token t of query block i, head h: causal softmax attention over
//           the tokens u <= t (u < L_b) of the kept blocks of (b, kvh, i)
//
// prefill_gate_kernel / prefill_select_kernel: one CTA per (row, query block).
// prefill_attn_kernel: one CTA per (b, query head, query block), the heads of
// a group launched side by side so they share K/V tiles through L2, 16 query
// rows per warp, FlashAttention-style online softmax on mma.sync (S = Q K^T
// and O += P V, the S accumulators re-packed as the A operand of P V), K/V
// tiles double-buffered in shared memory by cp.async; rows past L_b are
// zero-filled by the copy itself, so no cache padding reaches the math.
#include <cuda_bf16.h>

#include "gate_core.cuh"
#include "seer_launch.h"

namespace seer {
namespace {

constexpr int kGateThreads = 256;
constexpr int kGateWarps = kGateThreads / 32;
constexpr float kLog2e = 1.44269504088896340736f;
constexpr float kLn2 = 0.69314718055994530942f;

template <int D, int DG>
__global__ void __launch_bounds__(kGateThreads)
    prefill_gate_kernel(const __nv_bfloat16* __restrict__ q, const float* __restrict__ w_q,
                        const float* __restrict__ kpool, const int32_t* __restrict__ seq_lens, int Hq, int Hkv,
                        int Lmax, int blk, int NBmax, float* __restrict__ scores) {
    __shared__ __align__(16) float part[kGateThreads / D][D];
    __shared__ __align__(16) float qbar[D];
    __shared__ __align__(16) float qg[DG];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int i = blockIdx.x, row = blockIdx.y;
    const int b = row / Hkv, kvh = row - b * Hkv;
    const int G = Hq / Hkv;
    const int L = clamp_len(seq_lens[b], Lmax);
    const int NB = (L + blk - 1) / blk;
    if (i >= NB) return;
    const int t0 = i * blk, t1 = min(t0 + blk, L);
    // group- and block-mean of the queries: thread (d, p) sums tokens t0 + p, t0 + p + P, ...
    constexpr int P = kGateThreads / D;
    {
        const int d = tid % D, p = tid / D;
        float acc = 0.f;
        for (int h = 0; h < G; ++h) {
            const __nv_bfloat16* qh = q + (((size_t)b * Hq + (size_t)kvh * G + h) * Lmax) * D + d;
            for (int t = t0 + p; t < t1; t += P) acc += __bfloat162float(qh[(size_t)t * D]);
        }
        part[p][d] = acc;
    }
    __syncthreads();
    if (tid < D) {
        float acc = 0.f;
        for (int p = 0; p < P; ++p) acc += part[p][tid];
        qbar[tid] = acc / (float)(G * (t1 - t0));
    }
    __syncthreads();
    const float* W = w_q + (size_t)kvh * DG * D;
    for (int e = warp; e < DG; e += kGateWarps) {
        float acc = 0.f;
#pragma unroll
        for (int u = 0; u < D / 32; ++u) acc = fmaf(W[(size_t)e * D + lane + 32 * u], qbar[lane + 32 * u], acc);
        acc = warp_sum(acc);
        if (lane == 0) qg[e] = acc;
    }
    __syncthreads();
    const float inv_sqrt_dg = 1.0f / sqrtf((float)DG);
    const float* kp = kpool + (size_t)row * NBmax * DG;
    float* out = scores + ((size_t)row * NBmax + i) * NBmax;
    const int quad = lane >> 2, qlane = lane & 3;
    for (int j0 = warp * 8; j0 <= i; j0 += kGateWarps * 8) {
        const int j = min(j0 + quad, i);
        const float d = quad_row_dot<DG>(kp + (size_t)j * DG, j, qg, qlane);
        if (qlane == 0 && j0 + quad <= i) out[j] = d * inv_sqrt_dg;
    }
}

constexpr int kSelThreads = 256;

__global__ void __launch_bounds__(kSelThreads)
    prefill_select_kernel(const float* __restrict__ scores, const int32_t* __restrict__ seq_lens, int Hkv, int Lmax,
                          int blk, int NBmax, int kmax, int32_t* __restrict__ block_idx,
                          int32_t* __restrict__ num_selected) {
    extern __shared__ uint32_t keys[];  // [NBmax]
    __shared__ SelectSmem<kSelThreads> sm;
    const int i = blockIdx.x, row = blockIdx.y;
    const int L = clamp_len(seq_lens[row / Hkv], Lmax);
    const int NB = (L + blk - 1) / blk;
    const int NBi = i < NB ? i + 1 : 0;  // query block i sees blocks 0 .. i; i is its "last" block
    const size_t ri = (size_t)row * NBmax + i;
    if (threadIdx.x == 0) num_selected[ri] = kmax < NBi ? kmax : NBi;
    const float* s = scores + ri * NBmax;
    for (int j = threadIdx.x; j < NBi - 1; j += kSelThreads) keys[j] = order_key(s[j]);
    __syncthreads();
    select_row<kSelThreads>(keys, NBi, kmax, block_idx + ri * kmax, sm);
}

template <int D, int BLK>
struct PrefillCfg {
    static constexpr int kWarps = BLK / 16;      // 16 query rows per warp
    static constexpr int kThreads = kWarps * 32;
    static constexpr int kRow = D * 2 + 16;      // padded tile row: conflict-free ldmatrix
    static constexpr int kTile = BLK * kRow;
    static constexpr int kSmem = 5 * kTile;      // Q, K x 2, V x 2
    static constexpr int kNT = BLK / 8;          // key n8 tiles per block
    static constexpr int kKS = D / 16;           // k16 steps over head_dim
    static constexpr int kDT = D / 8;            // head_dim n8 tiles of O
};

__device__ __forceinline__ void cp_async_commit_group() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void cp_async16_zfill(uint32_t dst, const void* src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
}

// All threads: rows 0 .. BLK-1 of the tile starting at token `t0` of `base`
// (token-major [*, D]); rows at or past `valid` are zero-filled without a read.
template <int D, int BLK>
__device__ __forceinline__ void load_rows(uint32_t dst, const __nv_bfloat16* base, int t0, int valid) {
    using C = PrefillCfg<D, BLK>;
    constexpr int kPer = D * 2 / 16;
    for (int c = threadIdx.x; c < BLK * kPer; c += C::kThreads) {
        const int r = c / kPer, q = c - r * kPer;
        const bool ok = r < valid;
        cp_async16_zfill(dst + r * C::kRow + q * 16, base + ((size_t)t0 + (ok ? r : 0)) * D + q * 8, ok);
    }
}

template <int D, int BLK>
__global__ void __launch_bounds__(PrefillCfg<D, BLK>::kThreads, 1)
    prefill_attn_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k_cache,
                        const __nv_bfloat16* __restrict__ v_cache, const int32_t* __restrict__ seq_lens,
                        const int32_t* __restrict__ block_idx, const int32_t* __restrict__ num_selected, int Hq,
                        int Hkv, int Lmax, int NBmax, int kmax, float scale_log2, __nv_bfloat16* __restrict__ out,
                        float* __restrict__ lse_out) {
    using C = PrefillCfg<D, BLK>;
    extern __shared__ __align__(16) unsigned char smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, tig = lane & 3;
    // blockIdx.x = query block * G + head of the group: the G heads reading the
    // same K/V tiles (and the next query blocks, which keep mostly the same
    // blocks) launch next to each other, so the tiles are shared through L2
    const int G = Hq / Hkv;
    const int i = blockIdx.x / G, row = blockIdx.y;
    const int b = row / Hkv, kvh = row - b * Hkv;
    const int hq = kvh * G + (blockIdx.x - i * G);
    const int bh = b * Hq + hq;
    const int L = clamp_len(seq_lens[b], Lmax);
    const int t0 = i * BLK;
    const int r0 = t0 + warp * 16 + g, r1 = r0 + 8;  // this lane's two query rows
    __nv_bfloat16* ob = out + (size_t)bh * Lmax * D;
    if (t0 >= L) {  // the whole query block is past the length: zero output, lse -inf
        for (int c = threadIdx.x; c < BLK * D; c += C::kThreads)
            if (t0 + c / D < Lmax) ob[(size_t)t0 * D + c] = __float2bfloat16(0.f);
        if (lse_out)
            for (int c = threadIdx.x; c < BLK; c += C::kThreads)
                if (t0 + c < Lmax) lse_out[(size_t)bh * Lmax + t0 + c] = -INFINITY;
        return;
    }
    const uint32_t sQ = smem_addr(smem), sK = sQ + C::kTile, sV = sK + 2 * C::kTile;
    const __nv_bfloat16* kb = k_cache + (size_t)row * Lmax * D;
    const __nv_bfloat16* vb = v_cache + (size_t)row * Lmax * D;
    const int32_t* list = block_idx + ((size_t)row * NBmax + i) * kmax;
    const int nsel = min(num_selected[(size_t)row * NBmax + i], kmax);

    load_rows<D, BLK>(sQ, q + (size_t)bh * Lmax * D, t0, L - t0);
    int x = 0;  // next list entry to load
    auto next_valid = [&](int from) {
        while (from < nsel && (list[from] < 0 || list[from] > i)) ++from;
        return from;
    };
    x = next_valid(0);
    if (x < nsel) {
        const int j = list[x];
        load_rows<D, BLK>(sK, kb, j * BLK, L - j * BLK);
        load_rows<D, BLK>(sV, vb, j * BLK, L - j * BLK);
    }
    cp_async_commit_group();

    float o[C::kDT][4];
#pragma unroll
    for (int dt = 0; dt < C::kDT; ++dt) o[dt][0] = o[dt][1] = o[dt][2] = o[dt][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    int stage = 0;
    while (x < nsel) {
        const int j = list[x];
        const int xn = next_valid(x + 1);
        if (xn < nsel) {  // prefetch the next kept block into the other stage
            const int jn = list[xn];
            load_rows<D, BLK>(sK + (stage ^ 1) * C::kTile, kb, jn * BLK, L - jn * BLK);
            load_rows<D, BLK>(sV + (stage ^ 1) * C::kTile, vb, jn * BLK, L - jn * BLK);
        }
        cp_async_commit_group();
        cp_async_wait_group<1>();
        __syncthreads();
        const uint32_t cK = sK + stage * C::kTile, cV = sV + stage * C::kTile;
        // ---- S = Q K^T for this warp's 16 rows
        float s[C::kNT][4];
#pragma unroll
        for (int nt = 0; nt < C::kNT; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
        for (int kk2 = 0; kk2 < C::kKS / 2; ++kk2) {
            uint32_t a[2][4];
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                const int kk = 2 * kk2 + h2;
                ldmatrix_x4(sQ + (warp * 16 + (lane & 15)) * C::kRow + (kk * 16 + (lane >> 4) * 8) * 2, a[h2][0],
                            a[h2][1], a[h2][2], a[h2][3]);
            }
#pragma unroll
            for (int nt = 0; nt < C::kNT; ++nt) {
                const int mi = lane >> 3;
                uint32_t b0, b1, b2, b3;
                ldmatrix_x4(cK + (nt * 8 + (lane & 7)) * C::kRow + ((2 * kk2 + (mi >> 1)) * 16 + (mi & 1) * 8) * 2, b0,
                            b1, b2, b3);
                mma_bf16_16816(s[nt], a[0][0], a[0][1], a[0][2], a[0][3], b0, b1);
                mma_bf16_16816(s[nt], a[1][0], a[1][1], a[1][2], a[1][3], b2, b3);
            }
        }
        // ---- mask (causal on the diagonal block, the sequence end) and online softmax
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < C::kNT; ++nt) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int u = j * BLK + nt * 8 + 2 * tig + e;
                const bool ok0 = u < L && (j < i || u <= r0);
                const bool ok1 = u < L && (j < i || u <= r1);
                s[nt][e] = ok0 ? s[nt][e] * scale_log2 : -INFINITY;
                s[nt][2 + e] = ok1 ? s[nt][2 + e] * scale_log2 : -INFINITY;
                mx0 = fmaxf(mx0, s[nt][e]);
                mx1 = fmaxf(mx1, s[nt][2 + e]);
            }
        }
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        const float n0 = fmaxf(m0, mx0), n1 = fmaxf(m1, mx1);
        const float u0 = n0 == -INFINITY ? 0.f : n0, u1 = n1 == -INFINITY ? 0.f : n1;
        const float al0 = exp2f(m0 - u0), al1 = exp2f(m1 - u1);
        m0 = n0;
        m1 = n1;
        l0 *= al0;
        l1 *= al1;
#pragma unroll
        for (int dt = 0; dt < C::kDT; ++dt) {
            o[dt][0] *= al0;
            o[dt][1] *= al0;
            o[dt][2] *= al1;
            o[dt][3] *= al1;
        }
#pragma unroll
        for (int nt = 0; nt < C::kNT; ++nt) {
            s[nt][0] = exp2f(s[nt][0] - u0);
            s[nt][1] = exp2f(s[nt][1] - u0);
            s[nt][2] = exp2f(s[nt][2] - u1);
            s[nt][3] = exp2f(s[nt][3] - u1);
            l0 += s[nt][0] + s[nt][1];
            l1 += s[nt][2] + s[nt][3];
        }
        // ---- O += P V (P re-packed from the S accumulators as the A operand)
#pragma unroll
        for (int kk = 0; kk < C::kNT / 2; ++kk) {
            const uint32_t a0 = pack_bf16x2(s[2 * kk][0], s[2 * kk][1]);
            const uint32_t a1 = pack_bf16x2(s[2 * kk][2], s[2 * kk][3]);
            const uint32_t a2 = pack_bf16x2(s[2 * kk + 1][0], s[2 * kk + 1][1]);
            const uint32_t a3 = pack_bf16x2(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
            for (int dp = 0; dp < C::kDT / 2; ++dp) {
                uint32_t b0, b1, b2, b3;
                const int key = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
                ldmatrix_x4_trans(cV + key * C::kRow + (dp * 16 + (lane >> 4) * 8) * 2, b0, b1, b2, b3);
                mma_bf16_16816(o[2 * dp], a0, a1, a2, a3, b0, b1);
                mma_bf16_16816(o[2 * dp + 1], a0, a1, a2, a3, b2, b3);
            }
        }
        __syncthreads();  // every warp is done with this stage before it is refilled
        stage ^= 1;
        x = xn;
    }
    cp_async_wait_group<0>();
    // ---- normalise and write this lane's two rows
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    const float i0 = l0 > 0.f ? 1.f / l0 : 0.f, i1 = l1 > 0.f ? 1.f / l1 : 0.f;
#pragma unroll
    for (int dt = 0; dt < C::kDT; ++dt) {
        const int d = dt * 8 + 2 * tig;
        if (r0 < Lmax)
            *reinterpret_cast<uint32_t*>(ob + (size_t)r0 * D + d) =
                r0 < L ? pack_bf16x2(o[dt][0] * i0, o[dt][1] * i0) : 0u;
        if (r1 < Lmax)
            *reinterpret_cast<uint32_t*>(ob + (size_t)r1 * D + d) =
                r1 < L ? pack_bf16x2(o[dt][2] * i1, o[dt][3] * i1) : 0u;
    }
    if (lse_out && tig == 0) {
        if (r0 < Lmax) lse_out[(size_t)bh * Lmax + r0] = (r0 < L && l0 > 0.f) ? (m0 + log2f(l0)) * kLn2 : -INFINITY;
        if (r1 < Lmax) lse_out[(size_t)bh * Lmax + r1] = (r1 < L && l1 > 0.f) ? (m1 + log2f(l1)) * kLn2 : -INFINITY;
    }
}

}  // namespace

cudaError_t launch_prefill_gate(const Shape& s, const void* q, const float* w_q, const float* kpool,
                                const int32_t* seq_lens, float* scores, cudaStream_t stream) {
    const auto* qb = static_cast<const __nv_bfloat16*>(q);
    const dim3 grid(s.NBmax, s.B * s.Hkv);
#define SEER_PG_CASE(DV, DGV)                                                                                      \
    if (s.D == DV && s.dg == DGV) {                                                                                \
        prefill_gate_kernel<DV, DGV><<<grid, kGateThreads, 0, stream>>>(qb, w_q, kpool, seq_lens, s.Hq, s.Hkv,    \
                                                                        s.Lmax, s.blk, s.NBmax, scores);          \
        return cudaGetLastError();                                                                                 \
    }
    SEER_PG_CASE(128, 128)
    SEER_PG_CASE(128, 64)
    SEER_PG_CASE(64, 128)
    SEER_PG_CASE(64, 64)
#undef SEER_PG_CASE
    return cudaErrorInvalidValue;
}

cudaError_t launch_prefill_select(const Shape& s, const float* scores, const int32_t* seq_lens, int kmax,
                                  int32_t* block_idx, int32_t* num_selected, cudaStream_t stream) {
    const size_t smem = (size_t)s.NBmax * sizeof(uint32_t);
    if (smem > 16 * 1024) {
        static bool attr_done = false;
        if (!attr_done) {
            cudaError_t e = cudaFuncSetAttribute(prefill_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 16384 * 4);
            if (e != cudaSuccess) return e;
            attr_done = true;
        }
    }
    prefill_select_kernel<<<dim3(s.NBmax, s.B * s.Hkv), kSelThreads, smem, stream>>>(
        scores, seq_lens, s.Hkv, s.Lmax, s.blk, s.NBmax, kmax, block_idx, num_selected);
    return cudaGetLastError();
}

template <int D, int BLK>
cudaError_t attn_impl(const Shape& s, const void* q, const void* k_cache, const void* v_cache, const int32_t* seq_lens,
                      const int32_t* block_idx, const int32_t* num_selected, int kmax, float sm_scale, void* out,
                      float* lse_out, cudaStream_t stream) {
    using C = PrefillCfg<D, BLK>;
    static bool attr_done = false;  // once per template instance (benign race)
    if (!attr_done) {
        cudaError_t e = cudaFuncSetAttribute(prefill_attn_kernel<D, BLK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             C::kSmem);
        if (e != cudaSuccess) return e;
        attr_done = true;
    }
    prefill_attn_kernel<D, BLK><<<dim3(s.NBmax * s.G, s.B * s.Hkv), C::kThreads, C::kSmem, stream>>>(
        static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k_cache),
        static_cast<const __nv_bfloat16*>(v_cache), seq_lens, block_idx, num_selected, s.Hq, s.Hkv, s.Lmax, s.NBmax,
        kmax, sm_scale * kLog2e, static_cast<__nv_bfloat16*>(out), lse_out);
    return cudaGetLastError();
}

cudaError_t launch_prefill_attention(const Shape& s, const void* q, const void* k_cache, const void* v_cache,
                                     const int32_t* seq_lens, const int32_t* block_idx, const int32_t* num_selected,
                                     int kmax, float sm_scale, void* out, float* lse_out, cudaStream_t stream) {
    if (s.D == 128 && s.blk == 64)
        return attn_impl<128, 64>(s, q, k_cache, v_cache, seq_lens, block_idx, num_selected, kmax, sm_scale, out,
                                  lse_out, stream);
    if (s.D == 128 && s.blk == 128)
        return attn_impl<128, 128>(s, q, k_cache, v_cache, seq_lens, block_idx, num_selected, kmax, sm_scale, out,
                                   lse_out, stream);
    if (s.D == 64 && s.blk == 64)
        return attn_impl<64, 64>(s, q, k_cache, v_cache, seq_lens, block_idx, num_selected, kmax, sm_scale, out,
                                 lse_out, stream);
    if (s.D == 64 && s.blk == 128)
        return attn_impl<64, 128>(s, q, k_cache, v_cache, seq_lens, block_idx, num_selected, kmax, sm_scale, out,
                                  lse_out, stream);
    return cudaErrorInvalidValue;
}

}  // namespace seer
