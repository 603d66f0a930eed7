// seer_api.cu -- the extern "C" entry points declared in include/seer.h:
// host-side validation, device-property lookup, TMA descriptor encoding, and
// the kernel launches. No allocation, no synchronisation, no state kept
// between calls beyond per-device constants (SM count) and the driver entry
// point of the tensor-map encoder.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdio>

#include "seer.h"
#include "seer_launch.h"

namespace {

using seer::Shape;

constexpr int kMaxDevices = 64;
int g_num_sms[kMaxDevices] = {0};

int device_sm_count() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return -1;
    if (dev < kMaxDevices && g_num_sms[dev] > 0) return g_num_sms[dev];
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return -1;
    if (dev < kMaxDevices) g_num_sms[dev] = n;
    return n;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Checks shared by every call; fills `s`.
seer_status check_dims(const seer_dims* d, Shape& s) {
    if (!d) return SEER_ERR_INVALID_ARG;
    if (d->batch < 1 || d->num_q_heads < 1 || d->num_kv_heads < 1 || d->max_seq_len < 1) return SEER_ERR_INVALID_ARG;
    if (d->num_q_heads % d->num_kv_heads != 0) return SEER_ERR_INVALID_ARG;
    const int G = d->num_q_heads / d->num_kv_heads;
    if (G > 8) return SEER_ERR_UNSUPPORTED;
    if (d->head_dim != 64 && d->head_dim != 128) return SEER_ERR_UNSUPPORTED;
    if (d->gate_dim != 64 && d->gate_dim != 128) return SEER_ERR_UNSUPPORTED;
    if (d->block_size != 64 && d->block_size != 128) return SEER_ERR_UNSUPPORTED;
    if (d->max_seq_len > (1 << 24)) return SEER_ERR_UNSUPPORTED;
    const long long rows = (long long)d->batch * d->num_kv_heads;
    if (rows > 65535) return SEER_ERR_UNSUPPORTED;
    if (rows * d->max_seq_len >= (1LL << 31)) return SEER_ERR_UNSUPPORTED;
    if ((long long)d->batch * d->num_q_heads >= (1LL << 31) / 128) return SEER_ERR_UNSUPPORTED;
    s.B = d->batch;
    s.Hq = d->num_q_heads;
    s.Hkv = d->num_kv_heads;
    s.G = G;
    s.D = d->head_dim;
    s.dg = d->gate_dim;
    s.blk = d->block_size;
    s.Lmax = d->max_seq_len;
    s.NBmax = (d->max_seq_len + d->block_size - 1) / d->block_size;
    return SEER_OK;
}

thread_local char g_last_error[256] = "no error";

seer_status from_cuda(cudaError_t e) {
    if (e == cudaSuccess) return SEER_OK;
    snprintf(g_last_error, sizeof(g_last_error), "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
    return SEER_ERR_CUDA;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// 2-D view [rows, D cols] of a bf16 tensor; box = 64 cols (128 B) x box_rows rows, 128-byte swizzle.
bool encode_rows_map(CUtensorMap* m, const void* base, int D, long long rows, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A bf16 cache [B*Hkv*Lmax rows, D cols] with a blk-row box.
bool encode_cache_map(CUtensorMap* m, const void* base, const Shape& s) {
    return encode_rows_map(m, base, s.D, (long long)s.B * s.Hkv * s.Lmax, s.blk);
}

}  // namespace

extern "C" {

seer_status seer_kpool_update(const seer_dims* dims, const void* k_cache, const float* w_k,
                              const int32_t* seq_lens, const int32_t* upd_start, float* kpool,
                              cudaStream_t stream) {
    Shape s;
    seer_status st = check_dims(dims, s);
    if (st != SEER_OK) return st;
    if (!k_cache || !w_k || !seq_lens || !kpool) return SEER_ERR_INVALID_ARG;
    if (!aligned(k_cache, 16) || !aligned(w_k, 16)) return SEER_ERR_INVALID_ARG;
    const int nsm = device_sm_count();
    if (nsm <= 0) return SEER_ERR_CUDA;
    return from_cuda(seer::launch_kpool_update(s, k_cache, w_k, seq_lens, upd_start, kpool, nsm, stream));
}

seer_status seer_gate_scores(const seer_dims* dims, const void* q, const float* w_q, const float* kpool,
                             const int32_t* seq_lens, float* scores, cudaStream_t stream) {
    Shape s;
    seer_status st = check_dims(dims, s);
    if (st != SEER_OK) return st;
    if (!q || !w_q || !kpool || !seq_lens || !scores) return SEER_ERR_INVALID_ARG;
    if (!aligned(w_q, 16) || !aligned(kpool, 16)) return SEER_ERR_INVALID_ARG;
    const int nsm = device_sm_count();
    if (nsm <= 0) return SEER_ERR_CUDA;
    return from_cuda(seer::launch_gate_scores(s, q, w_q, kpool, seq_lens, scores, nsm, stream));
}

seer_status seer_select_blocks(const seer_dims* dims, const float* scores, const int32_t* seq_lens,
                               int32_t budget_tokens, int32_t* block_idx, int32_t* num_selected,
                               cudaStream_t stream) {
    Shape s;
    seer_status st = check_dims(dims, s);
    if (st != SEER_OK) return st;
    if (!scores || !seq_lens || !block_idx || !num_selected) return SEER_ERR_INVALID_ARG;
    if (budget_tokens < s.blk || budget_tokens % s.blk != 0) return SEER_ERR_INVALID_ARG;
    if (s.NBmax > 16384) return SEER_ERR_UNSUPPORTED;
    return from_cuda(
        seer::launch_select_blocks(s, scores, seq_lens, budget_tokens / s.blk, block_idx, num_selected, stream));
}

seer_status seer_sparse_decode(const seer_dims* dims, const void* q, const void* k_cache, const void* v_cache,
                               const int32_t* seq_lens, const int32_t* block_idx, const int32_t* num_selected,
                               int32_t kmax, int32_t num_splits, float sm_scale, float* o_part, float* lse_part,
                               cudaStream_t stream) {
    Shape s;
    seer_status st = check_dims(dims, s);
    if (st != SEER_OK) return st;
    if (!q || !k_cache || !v_cache || !seq_lens || !block_idx || !num_selected || !o_part || !lse_part)
        return SEER_ERR_INVALID_ARG;
    if (kmax < 1 || num_splits < 1) return SEER_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16)) return SEER_ERR_INVALID_ARG;
    if (!(sm_scale == sm_scale) || std::isinf(sm_scale)) return SEER_ERR_INVALID_ARG;
    if ((long long)s.B * s.Hq * num_splits * s.D >= (1LL << 40)) return SEER_ERR_UNSUPPORTED;
    const int nsm = device_sm_count();
    if (nsm <= 0) return SEER_ERR_CUDA;
    CUtensorMap tmk, tmv;
    if (!encode_cache_map(&tmk, k_cache, s) || !encode_cache_map(&tmv, v_cache, s)) return SEER_ERR_CUDA;
    seer::DecodeLaunch a;
    a.q = q;
    a.seq_lens = seq_lens;
    a.block_idx = block_idx;
    a.num_selected = num_selected;
    a.o_part = o_part;
    a.lse_part = lse_part;
    a.kmax = kmax;
    a.num_splits = num_splits;
    a.sm_scale = sm_scale > 0.f ? sm_scale : 1.0f / std::sqrt((float)s.D);
    return from_cuda(seer::launch_sparse_decode(s, a, tmk, tmv, nsm, stream));
}

seer_status seer_combine(const seer_dims* dims, const float* o_part, const float* lse_part, int32_t num_splits,
                         void* out, float* lse_out, cudaStream_t stream) {
    Shape s;
    seer_status st = check_dims(dims, s);
    if (st != SEER_OK) return st;
    if (!o_part || !lse_part || !out || num_splits < 1) return SEER_ERR_INVALID_ARG;
    if (!aligned(o_part, 16) || !aligned(out, 8)) return SEER_ERR_INVALID_ARG;
    return from_cuda(seer::launch_combine(s, o_part, lse_part, num_splits, out, lse_out, stream));
}

constexpr int kMaxPrefillBlocks = 4096;  // the prefill score matrix is NBmax x NBmax per row

seer_status seer_prefill_gate_scores(const seer_dims* dims, const void* q, const float* w_q, const float* kpool,
                                     const int32_t* seq_lens, float* scores, cudaStream_t stream) {
    Shape s;
    seer_status st = check_dims(dims, s);
    if (st != SEER_OK) return st;
    if (!q || !w_q || !kpool || !seq_lens || !scores) return SEER_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(w_q, 16) || !aligned(kpool, 16)) return SEER_ERR_INVALID_ARG;
    if (s.NBmax > kMaxPrefillBlocks || s.B * s.Hkv > 65535) return SEER_ERR_UNSUPPORTED;  // grid y = rows
    return from_cuda(seer::launch_prefill_gate(s, q, w_q, kpool, seq_lens, scores, stream));
}

seer_status seer_prefill_select_blocks(const seer_dims* dims, const float* scores, const int32_t* seq_lens,
                                       int32_t budget_tokens, int32_t* block_idx, int32_t* num_selected,
                                       cudaStream_t stream) {
    Shape s;
    seer_status st = check_dims(dims, s);
    if (st != SEER_OK) return st;
    if (!scores || !seq_lens || !block_idx || !num_selected) return SEER_ERR_INVALID_ARG;
    if (budget_tokens < s.blk || budget_tokens % s.blk != 0) return SEER_ERR_INVALID_ARG;
    if (s.NBmax > kMaxPrefillBlocks || s.B * s.Hkv > 65535) return SEER_ERR_UNSUPPORTED;  // grid y = rows
    return from_cuda(
        seer::launch_prefill_select(s, scores, seq_lens, budget_tokens / s.blk, block_idx, num_selected, stream));
}

seer_status seer_prefill_attention(const seer_dims* dims, const void* q, const void* k_cache, const void* v_cache,
                                   const int32_t* seq_lens, const int32_t* block_idx, const int32_t* num_selected,
                                   int32_t kmax, float sm_scale, void* out, float* lse_out, cudaStream_t stream) {
    Shape s;
    seer_status st = check_dims(dims, s);
    if (st != SEER_OK) return st;
    if (!q || !k_cache || !v_cache || !seq_lens || !block_idx || !num_selected || !out || kmax < 1)
        return SEER_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(out, 16))
        return SEER_ERR_INVALID_ARG;
    if (!(sm_scale == sm_scale) || std::isinf(sm_scale)) return SEER_ERR_INVALID_ARG;
    if (s.NBmax > kMaxPrefillBlocks || s.B * s.Hkv > 65535) return SEER_ERR_UNSUPPORTED;  // grid y = rows
    const float scale = sm_scale > 0.f ? sm_scale : 1.0f / std::sqrt((float)s.D);
    if ((long long)s.B * s.Hq * s.Lmax >= (1LL << 31)) return SEER_ERR_UNSUPPORTED;  // 32-bit TMA row coordinate
    CUtensorMap tmq, tmk, tmv;
    if (!encode_rows_map(&tmq, q, s.D, (long long)s.B * s.Hq * s.Lmax, s.blk) ||
        !encode_rows_map(&tmk, k_cache, s.D, (long long)s.B * s.Hkv * s.Lmax, 64) ||
        !encode_rows_map(&tmv, v_cache, s.D, (long long)s.B * s.Hkv * s.Lmax, 64))
        return SEER_ERR_CUDA;
    return from_cuda(seer::launch_prefill_attention(s, tmq, tmk, tmv, seq_lens, block_idx, num_selected, kmax, scale,
                                                    out, lse_out, stream));
}

seer_status seer_gate_scores_agg(const seer_dims* dims, const void* q, const float* w_q, const float* kpool,
                                 const int32_t* seq_lens, int32_t aggregation, float* scores, cudaStream_t stream) {
    Shape s;
    seer_status st = check_dims(dims, s);
    if (st != SEER_OK) return st;
    if (!q || !w_q || !kpool || !seq_lens || !scores) return SEER_ERR_INVALID_ARG;
    if (aggregation < SEER_AGG_MEAN || aggregation > SEER_AGG_SOFTMAX_MEAN) return SEER_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(w_q, 16) || !aligned(kpool, 16)) return SEER_ERR_INVALID_ARG;
    return from_cuda(
        seer::launch_gate_scores_agg(s, q, w_q, kpool, seq_lens, aggregation, scores, device_sm_count(), stream));
}

seer_status seer_select_blocks_threshold(const seer_dims* dims, const float* scores, const int32_t* seq_lens,
                                         int32_t budget_tokens, float threshold, int32_t* block_idx,
                                         int32_t* num_selected, cudaStream_t stream) {
    Shape s;
    seer_status st = check_dims(dims, s);
    if (st != SEER_OK) return st;
    if (!scores || !seq_lens || !block_idx || !num_selected) return SEER_ERR_INVALID_ARG;
    if (budget_tokens < s.blk || budget_tokens % s.blk != 0) return SEER_ERR_INVALID_ARG;
    if (threshold != threshold) return SEER_ERR_INVALID_ARG;  // NaN: no order against it
    if (s.NBmax > 16384) return SEER_ERR_UNSUPPORTED;
    return from_cuda(
        seer::launch_select_threshold(s, scores, seq_lens, budget_tokens / s.blk, threshold, block_idx, num_selected,
                                      stream));
}

seer_status seer_block_mass(const seer_dims* dims, const void* q, const void* k_cache, const int32_t* seq_lens,
                            float sm_scale, float* mass, float* lse_out, cudaStream_t stream) {
    Shape s;
    seer_status st = check_dims(dims, s);
    if (st != SEER_OK) return st;
    if (!q || !k_cache || !seq_lens || !mass) return SEER_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(mass, 4)) return SEER_ERR_INVALID_ARG;
    if (!(sm_scale == sm_scale) || std::isinf(sm_scale)) return SEER_ERR_INVALID_ARG;
    const float scale = sm_scale > 0.f ? sm_scale : 1.0f / std::sqrt((float)s.D);
    return from_cuda(seer::launch_block_mass(s, q, k_cache, seq_lens, scale, mass, lse_out, stream));
}

seer_status seer_append_kv(const seer_dims* dims, const void* k_new, const void* v_new, const int32_t* seq_lens,
                           void* k_cache, void* v_cache, cudaStream_t stream) {
    Shape s;
    seer_status st = check_dims(dims, s);
    if (st != SEER_OK) return st;
    if (!k_new || !v_new || !seq_lens || !k_cache || !v_cache) return SEER_ERR_INVALID_ARG;
    if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16))
        return SEER_ERR_INVALID_ARG;
    return from_cuda(seer::launch_append_kv(s, k_new, v_new, seq_lens, k_cache, v_cache, stream));
}

seer_status seer_decode_step_workspace_size(const seer_dims* dims, int32_t budget_tokens, size_t* bytes) {
    Shape s;
    seer_status st = check_dims(dims, s);
    if (st != SEER_OK) return st;
    if (!bytes || budget_tokens < s.blk || budget_tokens % s.blk != 0) return SEER_ERR_INVALID_ARG;
    const int nsm = device_sm_count();
    if (nsm <= 0) return SEER_ERR_CUDA;
    *bytes = seer::step_workspace_layout(s, budget_tokens / s.blk, nsm).total;
    return SEER_OK;
}

seer_status seer_decode_step(const seer_dims* dims, const void* q, const void* k_cache, const void* v_cache,
                             const float* w_q, const float* w_k, const int32_t* seq_lens, const int32_t* upd_start,
                             int32_t budget_tokens, float sm_scale, float* kpool, int32_t* block_idx,
                             int32_t* num_selected, void* out, float* lse_out, void* workspace,
                             size_t workspace_bytes, cudaStream_t stream) {
    Shape s;
    seer_status st = check_dims(dims, s);
    if (st != SEER_OK) return st;
    if (!q || !k_cache || !v_cache || !w_q || !w_k || !seq_lens || !kpool || !block_idx || !num_selected || !out ||
        !workspace)
        return SEER_ERR_INVALID_ARG;
    if (budget_tokens < s.blk || budget_tokens % s.blk != 0) return SEER_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(w_q, 16) ||
        !aligned(w_k, 16) || !aligned(kpool, 16) || !aligned(workspace, 256) || !aligned(out, 2))
        return SEER_ERR_INVALID_ARG;
    if (!(sm_scale == sm_scale) || std::isinf(sm_scale)) return SEER_ERR_INVALID_ARG;
    if (s.NBmax > 16384) return SEER_ERR_UNSUPPORTED;
    const int nsm = device_sm_count();
    if (nsm <= 0) return SEER_ERR_CUDA;
    if (workspace_bytes < seer::step_workspace_layout(s, budget_tokens / s.blk, nsm).total)
        return SEER_ERR_INVALID_ARG;
    CUtensorMap tmk, tmv;
    if (!encode_cache_map(&tmk, k_cache, s) || !encode_cache_map(&tmv, v_cache, s)) return SEER_ERR_CUDA;
    seer::StepLaunch a;
    a.q = q;
    a.k_cache = k_cache;
    a.v_cache = v_cache;
    a.w_q = w_q;
    a.w_k = w_k;
    a.seq_lens = seq_lens;
    a.upd_start = upd_start;
    a.budget_tokens = budget_tokens;
    a.sm_scale = sm_scale > 0.f ? sm_scale : 1.0f / std::sqrt((float)s.D);
    a.kpool = kpool;
    a.block_idx = block_idx;
    a.num_selected = num_selected;
    a.out = out;
    a.lse_out = lse_out;
    a.workspace = workspace;
    return from_cuda(seer::launch_decode_step(s, a, tmk, tmv, nsm, stream));
}

seer_status seer_decode_step_noalloc(const seer_dims* dims, const void* q, const void* k_cache, const void* v_cache,
                                     const float* w_q, const float* w_k, const int32_t* seq_lens,
                                     const int32_t* upd_start, int32_t budget_tokens, float sm_scale, float* kpool,
                                     int32_t* block_idx, int32_t* num_selected, void* out, float* lse_out,
                                     cudaStream_t stream) {
    Shape s;
    seer_status st = check_dims(dims, s);
    if (st != SEER_OK) return st;
    if (!q || !k_cache || !v_cache || !w_q || !w_k || !seq_lens || !kpool || !block_idx || !num_selected || !out)
        return SEER_ERR_INVALID_ARG;
    if (budget_tokens < s.blk || budget_tokens % s.blk != 0) return SEER_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(w_q, 16) ||
        !aligned(w_k, 16) || !aligned(kpool, 16) || !aligned(out, 2))
        return SEER_ERR_INVALID_ARG;
    if (!(sm_scale == sm_scale) || std::isinf(sm_scale)) return SEER_ERR_INVALID_ARG;
    if (s.NBmax > 16384) return SEER_ERR_UNSUPPORTED;
    const int nsm = device_sm_count();
    if (nsm <= 0) return SEER_ERR_CUDA;
    if (seer::step_workspace_layout(s, budget_tokens / s.blk, nsm).total > seer::static_scratch_bytes()) {
        snprintf(g_last_error, sizeof(g_last_error),
                 "seer_decode_step_noalloc: scratch for these sizes exceeds the %zu-byte static array; use "
                 "seer_decode_step with a workspace", seer::static_scratch_bytes());
        return SEER_ERR_UNSUPPORTED;
    }
    CUtensorMap tmk, tmv;
    if (!encode_cache_map(&tmk, k_cache, s) || !encode_cache_map(&tmv, v_cache, s)) return SEER_ERR_CUDA;
    seer::StepLaunch a;
    a.q = q;
    a.k_cache = k_cache;
    a.v_cache = v_cache;
    a.w_q = w_q;
    a.w_k = w_k;
    a.seq_lens = seq_lens;
    a.upd_start = upd_start;
    a.budget_tokens = budget_tokens;
    a.sm_scale = sm_scale > 0.f ? sm_scale : 1.0f / std::sqrt((float)s.D);
    a.kpool = kpool;
    a.block_idx = block_idx;
    a.num_selected = num_selected;
    a.out = out;
    a.lse_out = lse_out;
    a.workspace = nullptr;
    return from_cuda(seer::launch_decode_step_static(s, a, tmk, tmv, nsm, stream));
}

seer_status seer_default_num_splits(int32_t kmax, int32_t* num_splits) {
    if (kmax < 1 || !num_splits) return SEER_ERR_INVALID_ARG;
    const int nsm = device_sm_count();
    if (nsm <= 0) return SEER_ERR_CUDA;
    *num_splits = kmax < nsm ? kmax : nsm;
    return SEER_OK;
}

seer_status seer_decode_wait_failures(uint32_t* count, int32_t reset) {
    if (!count) return SEER_ERR_INVALID_ARG;
    unsigned int c = 0;
    if (seer::read_decode_wait_failures(&c, reset != 0) != cudaSuccess) return SEER_ERR_CUDA;
    *count = c;
    return SEER_OK;
}

seer_status seer_wait_selftest(int64_t limit_ns, int32_t* timed_out) {
    if (!timed_out || limit_ns < 0 || limit_ns > 2000000000LL) return SEER_ERR_INVALID_ARG;
    int r = -1;
    if (seer::run_wait_selftest((unsigned long long)limit_ns, &r) != cudaSuccess) return SEER_ERR_CUDA;
    *timed_out = r;
    return SEER_OK;
}

const char* seer_last_error_string(void) { return g_last_error; }

const char* seer_status_string(seer_status status) {
    switch (status) {
        case SEER_OK: return "ok";
        case SEER_ERR_INVALID_ARG: return "invalid argument";
        case SEER_ERR_UNSUPPORTED: return "unsupported size";
        case SEER_ERR_CUDA: return "CUDA error";
    }
    return "unknown status";
}

}  // extern "C"
