// attn_api.cu -- the C ABI declared in include/attn.h: argument validation on the host,
// TMA descriptor encoding, dispatch to the kernels, and the per-device error word.
#include <cudaTypedefs.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <mutex>
#include <vector>

#include "../../include/attn.h"
#include "kernels.h"
#include "sm100.cuh"

namespace attn {

__device__ uint32_t g_device_error = 0;
__device__ uint64_t g_wait_limit_ns = kDefaultWaitLimitNs;

namespace {

thread_local char g_last_error[256] = {0};

attn_status fail(attn_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
  va_end(ap);
  return st;
}

attn_status ok() {
  g_last_error[0] = 0;
  return ATTN_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shared validation of the shape arguments; fills `pb`.
attn_status check_shapes(const int32_t* cu_seqlens, int32_t batch, int32_t seqlen, int32_t max_seqlen,
                         int32_t total_tokens, int32_t hq, int32_t hkv, int32_t d, float scale, int32_t causal,
                         int32_t dtype, Problem* pb) {
  if (dtype != ATTN_BF16 && dtype != ATTN_FP32) return fail(ATTN_ERR_UNSUPPORTED, "dtype %d is not supported", dtype);
  if (d != 32 && d != 64 && d != 128) return fail(ATTN_ERR_UNSUPPORTED, "head dim %d not in {32, 64, 128}", d);
  if (hq <= 0 || hkv <= 0) return fail(ATTN_ERR_INVALID_ARG, "head counts must be positive (hq=%d hkv=%d)", hq, hkv);
  if (hq % hkv != 0) return fail(ATTN_ERR_UNSUPPORTED, "hq=%d is not a multiple of hkv=%d", hq, hkv);
  if (hq > 65535 || batch > 65535) return fail(ATTN_ERR_UNSUPPORTED, "hq and batch must be <= 65535");
  if (batch < 0 || total_tokens < 0 || max_seqlen < 0)
    return fail(ATTN_ERR_INVALID_ARG, "negative batch / total_tokens / max_seqlen");
  if (!(scale > 0.f) || !isfinite(scale)) return fail(ATTN_ERR_INVALID_ARG, "scale must be positive and finite");
  if (causal != 0 && causal != 1) return fail(ATTN_ERR_INVALID_ARG, "causal must be 0 or 1");
  if (cu_seqlens == nullptr) {
    if (seqlen < 0) return fail(ATTN_ERR_INVALID_ARG, "negative seqlen");
    if ((int64_t)batch * seqlen != total_tokens)
      return fail(ATTN_ERR_INVALID_ARG, "batch mode needs total_tokens == batch * seqlen (%d * %d != %d)", batch,
                  seqlen, total_tokens);
    max_seqlen = seqlen;
  } else {
    if (!aligned16(cu_seqlens) && (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u))
      return fail(ATTN_ERR_INVALID_ARG, "cu_seqlens is not 4-byte aligned");
    if (max_seqlen > total_tokens) return fail(ATTN_ERR_INVALID_ARG, "max_seqlen > total_tokens");
  }
  // TMA row coordinates and the [hq, T] statistics are addressed with 32-bit rows.
  if ((int64_t)total_tokens * hq > (int64_t)INT32_MAX * 4)
    return fail(ATTN_ERR_UNSUPPORTED, "problem too large for this library");
  pb->cu_seqlens = cu_seqlens;
  pb->batch = batch;
  pb->seqlen = cu_seqlens ? 0 : seqlen;
  pb->max_seqlen = max_seqlen;
  pb->total_tokens = total_tokens;
  pb->hq = hq;
  pb->hkv = hkv;
  pb->d = d;
  pb->scale = scale;
  pb->causal = causal;
  return ATTN_OK;
}

attn_status check_ptr(const void* p, const char* name) {
  if (p == nullptr) return fail(ATTN_ERR_INVALID_ARG, "%s is NULL", name);
  if (!aligned16(p)) return fail(ATTN_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
  return ATTN_OK;
}

attn_status from_cuda(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return ok();
  return fail(ATTN_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// ---- launch bookkeeping ---------------------------------------------------------------
struct EventPair {
  cudaEvent_t start = nullptr, end = nullptr;
  int kind = 0;
};
std::mutex g_prof_mu;
bool g_prof_on = false;
std::vector<EventPair> g_prof_pool;      // created events, reused
std::vector<int> g_prof_pending;         // indices into the pool recorded since the last collect
std::vector<int> g_prof_free;            // indices free for reuse
std::atomic<int64_t> g_launches{0};

}  // namespace

int validate_shapes(const int32_t* cu_seqlens, int32_t batch, int32_t seqlen, int32_t max_seqlen, int32_t total_tokens,
                    int32_t hq, int32_t hkv, int32_t d, float scale, int32_t causal, int32_t dtype, Problem* pb) {
  return check_shapes(cu_seqlens, batch, seqlen, max_seqlen, total_tokens, hq, hkv, d, scale, causal, dtype, pb);
}
int validate_ptr(const void* p, const char* name) { return check_ptr(p, name); }
int cuda_status(cudaError_t e, const char* what) { return from_cuda(e, what); }
int status_ok() { return ok(); }

int record_error(int status, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
  va_end(ap);
  return status;
}

const char* kernel_kind_name(int kind) {
  static const char* names[K_NUM_KINDS] = {"fwd_bf16_sm100",  "bwd_preprocess",       "bwd_bf16_sm100",
                                           "bwd_dq_convert",  "fwd_fp32_kernel",      "bwd_fp32_dq_kernel",
                                           "bwd_fp32_dkdv_kernel", "decode_bf16_sm100", "decode_combine",
                                           "merge_partial",   "merge_finish",         "fwd_fp8_sm100",
                                           "fp8_quantize",    "selftest"};
  return (kind >= 0 && kind < K_NUM_KINDS) ? names[kind] : "";
}

LaunchScope::LaunchScope(int k, cudaStream_t s) : kind(k), stream(s), slot(-1) {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (!g_prof_on) return;
  int idx;
  if (!g_prof_free.empty()) {
    idx = g_prof_free.back();
    g_prof_free.pop_back();
  } else {
    EventPair ep;
    if (cudaEventCreate(&ep.start) != cudaSuccess || cudaEventCreate(&ep.end) != cudaSuccess) return;
    g_prof_pool.push_back(ep);
    idx = (int)g_prof_pool.size() - 1;
  }
  g_prof_pool[idx].kind = kind;
  if (cudaEventRecord(g_prof_pool[idx].start, stream) != cudaSuccess) {
    g_prof_free.push_back(idx);
    return;
  }
  slot = idx;
}

LaunchScope::~LaunchScope() {
  if (slot < 0) return;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (cudaEventRecord(g_prof_pool[slot].end, stream) == cudaSuccess)
    g_prof_pending.push_back(slot);
  else
    g_prof_free.push_back(slot);
}

bool encode_tma_3d(void* tmap_out, const void* base, int d, int heads, int rows, int box_inner, int box_rows) {
  return encode_tma_3d_box(tmap_out, base, d, heads, rows, box_inner, 1, box_rows);
}

bool encode_tma_3d_box(void* tmap_out, const void* base, int d, int heads, int rows, int box_inner, int box_heads,
                       int box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = encoder();
  if (!enc) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)heads, (cuuint64_t)rows};
  const cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)heads * d * 2};
  const cuuint32_t box[3] = {(cuuint32_t)box_inner, (cuuint32_t)box_heads, (cuuint32_t)box_rows};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  const CUtensorMapSwizzle swz = box_inner * 2 == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                 : box_inner * 2 == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                       : CU_TENSOR_MAP_SWIZZLE_NONE;
  CUresult r = enc(reinterpret_cast<CUtensorMap*>(tmap_out), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                   const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_tma_u8_3d(void* tmap_out, const void* base, int dim0, int dim1, int dim2, uint64_t stride1,
                      uint64_t stride2, int box0, int box1, int box2) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = encoder();
  if (!enc) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)dim0, (cuuint64_t)dim1, (cuuint64_t)dim2};
  const cuuint64_t strides[2] = {(cuuint64_t)stride1, (cuuint64_t)stride2};
  const cuuint32_t box[3] = {(cuuint32_t)box0, (cuuint32_t)box1, (cuuint32_t)box2};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = enc(reinterpret_cast<CUtensorMap*>(tmap_out), CU_TENSOR_MAP_DATA_TYPE_UINT8, 3,
                   const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   box0 == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                   : box0 == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                : CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_tma_3d_f32(void* tmap_out, const void* base, int d, int heads, int rows, int box_inner, int box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = encoder();
  if (!enc) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)heads, (cuuint64_t)rows};
  const cuuint64_t strides[2] = {(cuuint64_t)d * 4, (cuuint64_t)heads * d * 4};
  const cuuint32_t box[3] = {(cuuint32_t)box_inner, 1u, (cuuint32_t)box_rows};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = enc(reinterpret_cast<CUtensorMap*>(tmap_out), CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3,
                   const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   box_inner * 4 == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace attn

using namespace attn;

namespace {
// Shapes of the FP8 calls: a fixed-length batch (cu_seqlens NULL: batch sequences of seqlen
// tokens) or packed sequences (cu_seqlens, max_seqlen, total_tokens); d = 64 or 128.
attn_status check_fp8(const int32_t* cu_seqlens, int32_t batch, int32_t seqlen, int32_t max_seqlen,
                      int32_t total_tokens, int32_t hq, int32_t hkv, int32_t d, float scale, int32_t causal,
                      Problem* pb) {
  if (d != 64 && d != 128) return fail(ATTN_ERR_UNSUPPORTED, "the FP8 forward needs head dim 64 or 128 (got %d)", d);
  if (batch < 0 || seqlen < 0 || max_seqlen < 0 || total_tokens < 0)
    return fail(ATTN_ERR_INVALID_ARG, "negative batch / seqlen / max_seqlen / total_tokens");
  if (cu_seqlens == nullptr) {
    if ((int64_t)batch * seqlen > INT32_MAX) return fail(ATTN_ERR_UNSUPPORTED, "problem too large for this library");
    max_seqlen = seqlen;
    total_tokens = batch * seqlen;
  }
  if ((int64_t)batch * hkv > 65535) return fail(ATTN_ERR_UNSUPPORTED, "batch * hkv must be <= 65535");
  if ((int64_t)batch * hkv * d * fp8_vt_pitch(max_seqlen) > ((int64_t)1 << 40))
    return fail(ATTN_ERR_UNSUPPORTED, "problem too large for this library");
  return check_shapes(cu_seqlens, batch, seqlen, max_seqlen, total_tokens, hq, hkv, d, scale, causal, ATTN_BF16, pb);
}
}  // namespace

extern "C" {

attn_status attn_fwd(const void* q, const void* k, const void* v, const int32_t* cu_seqlens, int32_t batch,
                     int32_t seqlen, int32_t max_seqlen, int32_t total_tokens, int32_t hq, int32_t hkv, int32_t d,
                     float scale, int32_t causal, int32_t dtype, void* o, float* lse, void* workspace,
                     size_t workspace_bytes, void* stream) {
  Problem pb;
  attn_status st = check_shapes(cu_seqlens, batch, seqlen, max_seqlen, total_tokens, hq, hkv, d, scale, causal,
                                dtype, &pb);
  if (st != ATTN_OK) return st;
  if (total_tokens == 0 || batch == 0) return ok();
  if ((st = check_ptr(q, "q")) || (st = check_ptr(k, "k")) || (st = check_ptr(v, "v")) ||
      (st = check_ptr(o, "o")) || (st = check_ptr(lse, "lse")))
    return st;
  if (dtype == ATTN_BF16) {
    if (workspace_bytes < kFwdWorkspaceBytes)
      return fail(ATTN_ERR_INVALID_ARG, "workspace too small: %zu bytes given, %zu needed", workspace_bytes,
                  kFwdWorkspaceBytes);
    if ((st = check_ptr(workspace, "workspace"))) return st;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == ATTN_BF16)
    return from_cuda(launch_fwd_bf16(pb, q, k, v, o, lse, workspace, s), "attn_fwd launch");
  return from_cuda(launch_fwd_fp32(pb, static_cast<const float*>(q), static_cast<const float*>(k),
                                   static_cast<const float*>(v), static_cast<float*>(o), lse, s),
                   "attn_fwd (fp32 check mode) launch");
}

attn_status attn_fp8_quantize_varlen(const void* q, const void* k, const void* v, const int32_t* cu_seqlens,
                                     int32_t batch, int32_t max_seqlen, int32_t total_tokens, int32_t hq, int32_t hkv,
                                     int32_t d, void* q8, void* k8, void* vt8, float* descale_q, float* descale_k,
                                     float* descale_v, void* stream) {
  Problem pb;
  if (cu_seqlens == nullptr) return fail(ATTN_ERR_INVALID_ARG, "cu_seqlens is NULL");
  attn_status st = check_fp8(cu_seqlens, batch, 0, max_seqlen, total_tokens, hq, hkv, d, 1.f, 0, &pb);
  if (st != ATTN_OK) return st;
  if (batch == 0 || total_tokens == 0) return ok();
  if ((st = check_ptr(q, "q")) || (st = check_ptr(k, "k")) || (st = check_ptr(v, "v")) || (st = check_ptr(q8, "q8")) ||
      (st = check_ptr(k8, "k8")) || (st = check_ptr(vt8, "vt8")) || (st = check_ptr(descale_q, "descale_q")) ||
      (st = check_ptr(descale_k, "descale_k")) || (st = check_ptr(descale_v, "descale_v")))
    return st;
  return from_cuda(launch_fp8_quantize(q, k, v, cu_seqlens, batch, 0, max_seqlen, total_tokens, hq, hkv, d, q8, k8,
                                       vt8, descale_q, descale_k, descale_v, static_cast<cudaStream_t>(stream)),
                   "attn_fp8_quantize_varlen launch");
}

attn_status attn_fp8_quantize(const void* q, const void* k, const void* v, int32_t batch, int32_t seqlen, int32_t hq,
                              int32_t hkv, int32_t d, void* q8, void* k8, void* vt8, float* descale_q,
                              float* descale_k, float* descale_v, void* stream) {
  Problem pb;
  attn_status st = check_fp8(nullptr, batch, seqlen, 0, 0, hq, hkv, d, 1.f, 0, &pb);
  if (st != ATTN_OK) return st;
  if (batch == 0 || seqlen == 0) return ok();
  if ((st = check_ptr(q, "q")) || (st = check_ptr(k, "k")) || (st = check_ptr(v, "v")) || (st = check_ptr(q8, "q8")) ||
      (st = check_ptr(k8, "k8")) || (st = check_ptr(vt8, "vt8")) || (st = check_ptr(descale_q, "descale_q")) ||
      (st = check_ptr(descale_k, "descale_k")) || (st = check_ptr(descale_v, "descale_v")))
    return st;
  return from_cuda(launch_fp8_quantize(q, k, v, nullptr, batch, seqlen, seqlen, batch * seqlen, hq, hkv, d, q8, k8,
                                       vt8, descale_q, descale_k, descale_v, static_cast<cudaStream_t>(stream)),
                   "attn_fp8_quantize launch");
}

}  // extern "C"

namespace {
// The FP8 forward once the shapes are checked (pb) and the batch is not empty.
attn_status fwd_fp8_checked(const Problem& pb, const void* q8, const void* k8, const void* vt8,
                            const float* descale_q, const float* descale_k, const float* descale_v, void* o,
                            float* lse, void* workspace, size_t workspace_bytes, void* stream, const char* what) {
  attn_status st;
  if ((st = check_ptr(q8, "q8")) || (st = check_ptr(k8, "k8")) || (st = check_ptr(vt8, "vt8")) ||
      (st = check_ptr(descale_q, "descale_q")) || (st = check_ptr(descale_k, "descale_k")) ||
      (st = check_ptr(descale_v, "descale_v")) || (st = check_ptr(o, "o")) || (st = check_ptr(lse, "lse")))
    return st;
  if (workspace_bytes < kFwdWorkspaceBytes)
    return fail(ATTN_ERR_INVALID_ARG, "workspace too small: %zu bytes given, %zu needed", workspace_bytes,
                kFwdWorkspaceBytes);
  if ((st = check_ptr(workspace, "workspace"))) return st;
  return from_cuda(launch_fwd_fp8(pb, q8, k8, vt8, descale_q, descale_k, descale_v, o, lse, workspace,
                                  static_cast<cudaStream_t>(stream)),
                   what);
}
}  // namespace

extern "C" {

attn_status attn_fwd_fp8(const void* q8, const void* k8, const void* vt8, const float* descale_q,
                         const float* descale_k, const float* descale_v, int32_t batch, int32_t seqlen, int32_t hq,
                         int32_t hkv, int32_t d, float scale, int32_t causal, void* o, float* lse, void* workspace,
                         size_t workspace_bytes, void* stream) {
  Problem pb;
  attn_status st = check_fp8(nullptr, batch, seqlen, 0, 0, hq, hkv, d, scale, causal, &pb);
  if (st != ATTN_OK) return st;
  if (batch == 0 || seqlen == 0) return ok();
  return fwd_fp8_checked(pb, q8, k8, vt8, descale_q, descale_k, descale_v, o, lse, workspace, workspace_bytes, stream,
                         "attn_fwd_fp8 launch");
}

attn_status attn_fwd_fp8_varlen(const void* q8, const void* k8, const void* vt8, const float* descale_q,
                                const float* descale_k, const float* descale_v, const int32_t* cu_seqlens,
                                int32_t batch, int32_t max_seqlen, int32_t total_tokens, int32_t hq, int32_t hkv,
                                int32_t d, float scale, int32_t causal, void* o, float* lse, void* workspace,
                                size_t workspace_bytes, void* stream) {
  Problem pb;
  if (cu_seqlens == nullptr) return fail(ATTN_ERR_INVALID_ARG, "cu_seqlens is NULL");
  attn_status st = check_fp8(cu_seqlens, batch, 0, max_seqlen, total_tokens, hq, hkv, d, scale, causal, &pb);
  if (st != ATTN_OK) return st;
  if (batch == 0 || total_tokens == 0) return ok();
  return fwd_fp8_checked(pb, q8, k8, vt8, descale_q, descale_k, descale_v, o, lse, workspace, workspace_bytes, stream,
                         "attn_fwd_fp8_varlen launch");
}

}  // extern "C"

namespace {
// Validation of the decoding call's shape arguments; fills `pb`.
attn_status check_decode(const int32_t* cu_q, const int32_t* cu_k, int32_t batch, int32_t seqlen_q,
                         int32_t seqlen_k, int32_t max_seqlen_q, int32_t max_seqlen_k, int32_t total_q,
                         int32_t total_k, int32_t hq, int32_t hkv, int32_t d, float scale, int32_t causal,
                         int32_t num_splits, DecodeProblem* pb) {
  if (d != 32 && d != 64 && d != 128) return fail(ATTN_ERR_UNSUPPORTED, "head dim %d not in {32, 64, 128}", d);
  if (hq <= 0 || hkv <= 0) return fail(ATTN_ERR_INVALID_ARG, "head counts must be positive (hq=%d hkv=%d)", hq, hkv);
  if (hq % hkv != 0) return fail(ATTN_ERR_UNSUPPORTED, "hq=%d is not a multiple of hkv=%d", hq, hkv);
  if (hkv > 65535 || batch > 65535) return fail(ATTN_ERR_UNSUPPORTED, "hkv and batch must be <= 65535");
  if (batch < 0 || total_q < 0 || total_k < 0 || num_splits < 0)
    return fail(ATTN_ERR_INVALID_ARG, "negative batch / total_q / total_k / num_splits");
  if (!(scale > 0.f) || !isfinite(scale)) return fail(ATTN_ERR_INVALID_ARG, "scale must be positive and finite");
  if (causal != 0 && causal != 1) return fail(ATTN_ERR_INVALID_ARG, "causal must be 0 or 1");
  if ((cu_q == nullptr) != (cu_k == nullptr))
    return fail(ATTN_ERR_INVALID_ARG, "cu_seqlens_q and cu_seqlens_k must both be given or both be NULL");
  if (cu_q == nullptr) {
    if (seqlen_q < 0 || seqlen_k < 0) return fail(ATTN_ERR_INVALID_ARG, "negative seqlen_q / seqlen_k");
    if ((int64_t)batch * seqlen_q != total_q || (int64_t)batch * seqlen_k != total_k)
      return fail(ATTN_ERR_INVALID_ARG, "batch mode needs total_q == batch * seqlen_q and total_k == batch * seqlen_k");
    max_seqlen_q = seqlen_q;
    max_seqlen_k = seqlen_k;
  } else {
    if ((reinterpret_cast<uintptr_t>(cu_q) & 3u) || (reinterpret_cast<uintptr_t>(cu_k) & 3u))
      return fail(ATTN_ERR_INVALID_ARG, "cu_seqlens_q / cu_seqlens_k are not 4-byte aligned");
    if (max_seqlen_q < 0 || max_seqlen_k < 0 || max_seqlen_q > total_q || max_seqlen_k > total_k)
      return fail(ATTN_ERR_INVALID_ARG, "max_seqlen_q / max_seqlen_k out of range");
  }
  // one KV head's query rows (its hq/hkv heads x the newest max_seqlen_q tokens) share one
  // 128-row tile
  if ((int64_t)(hq / hkv) * max_seqlen_q > 128)
    return fail(ATTN_ERR_UNSUPPORTED, "(hq / hkv) * max_seqlen_q = %lld exceeds 128 query rows per KV head",
                (long long)(hq / hkv) * max_seqlen_q);
  if ((int64_t)total_q * hq > (int64_t)INT32_MAX || (int64_t)total_k * hkv > (int64_t)INT32_MAX * 4)
    return fail(ATTN_ERR_UNSUPPORTED, "problem too large for this library");
  pb->cu_q = cu_q;
  pb->cu_k = cu_k;
  pb->batch = batch;
  pb->seqlen_q = cu_q ? 0 : seqlen_q;
  pb->seqlen_k = cu_q ? 0 : seqlen_k;
  pb->max_seqlen_q = max_seqlen_q;
  pb->max_seqlen_k = max_seqlen_k;
  pb->total_q = total_q;
  pb->total_k = total_k;
  pb->hq = hq;
  pb->hkv = hkv;
  pb->d = d;
  pb->scale = scale;
  pb->causal = causal;
  pb->num_splits = num_splits;
  pb->varlen = cu_q != nullptr;
  return ATTN_OK;
}
}  // namespace

extern "C" {

attn_status attn_fwd_decode(const void* q, const void* k, const void* v, const int32_t* cu_seqlens_q,
                            const int32_t* cu_seqlens_k, int32_t batch, int32_t seqlen_q, int32_t seqlen_k,
                            int32_t max_seqlen_q, int32_t max_seqlen_k, int32_t total_q, int32_t total_k,
                            int32_t hq, int32_t hkv, int32_t d, float scale, int32_t causal, int32_t num_splits,
                            void* o, float* lse, void* workspace, size_t workspace_bytes, void* stream) {
  DecodeProblem pb;
  attn_status st = check_decode(cu_seqlens_q, cu_seqlens_k, batch, seqlen_q, seqlen_k, max_seqlen_q, max_seqlen_k,
                                total_q, total_k, hq, hkv, d, scale, causal, num_splits, &pb);
  if (st != ATTN_OK) return st;
  if (total_q == 0 || batch == 0) return ok();
  if ((st = check_ptr(q, "q")) || (st = check_ptr(o, "o")) || (st = check_ptr(lse, "lse"))) return st;
  if (total_k > 0 && ((st = check_ptr(k, "k")) || (st = check_ptr(v, "v")))) return st;
  const DecodeSplit sp = decode_split(pb);
  if (sp.workspace_bytes > 0) {
    if (workspace_bytes < sp.workspace_bytes)
      return fail(ATTN_ERR_INVALID_ARG, "workspace too small: %zu bytes given, %zu needed", workspace_bytes,
                  sp.workspace_bytes);
    if ((st = check_ptr(workspace, "workspace"))) return st;
  }
  // An empty key tensor still needs valid TMA descriptors: point them at q (never read).
  const void* kk = total_k > 0 ? k : q;
  const void* vv = total_k > 0 ? v : q;
  if (total_k == 0) pb.total_k = 1;
  return from_cuda(launch_decode_bf16(pb, q, kk, vv, o, lse, workspace, static_cast<cudaStream_t>(stream)),
                   "decode launch");
}

attn_status attn_merge_partial(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part,
                               int32_t total_tokens, int32_t hq, int32_t d, int32_t first, void* stream) {
  if (d != 32 && d != 64 && d != 128) return fail(ATTN_ERR_UNSUPPORTED, "head dim %d not in {32, 64, 128}", d);
  if (total_tokens < 0 || hq <= 0) return fail(ATTN_ERR_INVALID_ARG, "need total_tokens >= 0 and hq > 0");
  if (first != 0 && first != 1) return fail(ATTN_ERR_INVALID_ARG, "first must be 0 or 1");
  if ((int64_t)total_tokens * hq > (int64_t)INT32_MAX) return fail(ATTN_ERR_UNSUPPORTED, "problem too large");
  if (total_tokens == 0) return ok();
  attn_status st;
  if ((st = check_ptr(o_acc, "o_acc")) || (st = check_ptr(lse_acc, "lse_acc")) || (st = check_ptr(o_part, "o_part")) ||
      (st = check_ptr(lse_part, "lse_part")))
    return st;
  return from_cuda(launch_merge_partial(o_acc, lse_acc, o_part, lse_part, total_tokens, hq, d, first,
                                        static_cast<cudaStream_t>(stream)),
                   "merge launch");
}

attn_status attn_merge_finish(const float* o_acc, void* o, int32_t total_tokens, int32_t hq, int32_t d,
                              void* stream) {
  if (d != 32 && d != 64 && d != 128) return fail(ATTN_ERR_UNSUPPORTED, "head dim %d not in {32, 64, 128}", d);
  if (total_tokens < 0 || hq <= 0) return fail(ATTN_ERR_INVALID_ARG, "need total_tokens >= 0 and hq > 0");
  if ((int64_t)total_tokens * hq > (int64_t)INT32_MAX) return fail(ATTN_ERR_UNSUPPORTED, "problem too large");
  if (total_tokens == 0) return ok();
  attn_status st;
  if ((st = check_ptr(o_acc, "o_acc")) || (st = check_ptr(o, "o"))) return st;
  return from_cuda(launch_merge_finish(o_acc, o, total_tokens, hq, d, static_cast<cudaStream_t>(stream)),
                   "merge launch");
}

size_t attn_fwd_decode_workspace_size(int32_t batch, int32_t max_seqlen_q, int32_t max_seqlen_k, int32_t total_q,
                                      int32_t total_k, int32_t hq, int32_t hkv, int32_t d, int32_t varlen,
                                      int32_t num_splits) {
  if (batch <= 0 || total_q <= 0 || hq <= 0 || hkv <= 0 || d <= 0) return 0;
  DecodeProblem pb{};
  pb.batch = batch;
  pb.max_seqlen_q = max_seqlen_q;
  pb.max_seqlen_k = max_seqlen_k;
  pb.total_q = total_q;
  pb.total_k = total_k;
  pb.hq = hq;
  pb.hkv = hkv;
  pb.d = d;
  pb.varlen = varlen != 0;
  pb.num_splits = num_splits;
  return decode_split(pb).workspace_bytes;
}

size_t attn_fwd_workspace_size(int32_t batch, int32_t max_seqlen, int32_t total_tokens, int32_t hq, int32_t hkv,
                               int32_t d, int32_t dtype) {
  (void)batch, (void)max_seqlen, (void)hq, (void)hkv, (void)d;
  return (dtype == ATTN_BF16 && total_tokens > 0) ? kFwdWorkspaceBytes : 0;   // the work-item counter
}

size_t attn_bwd_workspace_size(int32_t batch, int32_t max_seqlen, int32_t total_tokens, int32_t hq, int32_t hkv,
                               int32_t d, int32_t dtype) {
  Problem pb{};
  pb.batch = batch;
  pb.max_seqlen = max_seqlen;
  pb.total_tokens = total_tokens;
  pb.hq = hq;
  pb.hkv = hkv;
  pb.d = d;
  if (total_tokens <= 0 || hq <= 0) return 0;
  return dtype == ATTN_FP32 ? bwd_fp32_workspace_bytes(pb) : bwd_bf16_workspace_bytes(pb);
}

}  // extern "C"

namespace attn {
// Host validation of the backward's arguments (shapes, then tensor pointers when there is
// work to do); touches no GPU state.
int bwd_check_args(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                   const int32_t* cu_seqlens, int32_t batch, int32_t seqlen, int32_t max_seqlen,
                   int32_t total_tokens, int32_t hq, int32_t hkv, int32_t d, float scale, int32_t causal,
                   int32_t dtype, void* dq, void* dk, void* dv, Problem* pb) {
  attn_status st = check_shapes(cu_seqlens, batch, seqlen, max_seqlen, total_tokens, hq, hkv, d, scale, causal,
                                dtype, pb);
  if (st != ATTN_OK) return st;
  if (total_tokens == 0 || batch == 0) return ok();
  if ((st = check_ptr(q, "q")) || (st = check_ptr(k, "k")) || (st = check_ptr(v, "v")) ||
      (st = check_ptr(o, "o")) || (st = check_ptr(dout, "dout")) || (st = check_ptr(lse, "lse")) ||
      (st = check_ptr(dq, "dq")) || (st = check_ptr(dk, "dk")) || (st = check_ptr(dv, "dv")))
    return st;
  return ok();
}
}  // namespace attn

extern "C" {

attn_status attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                     const int32_t* cu_seqlens, int32_t batch, int32_t seqlen, int32_t max_seqlen,
                     int32_t total_tokens, int32_t hq, int32_t hkv, int32_t d, float scale, int32_t causal,
                     int32_t dtype, void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes,
                     void* stream) {
  Problem pb;
  attn_status st = (attn_status)bwd_check_args(q, k, v, o, dout, lse, cu_seqlens, batch, seqlen, max_seqlen,
                                               total_tokens, hq, hkv, d, scale, causal, dtype, dq, dk, dv, &pb);
  if (st != ATTN_OK) return st;
  if (total_tokens == 0 || batch == 0) return ok();
  const size_t need = attn_bwd_workspace_size(batch, pb.max_seqlen, total_tokens, hq, hkv, d, dtype);
  if (workspace_bytes < need)
    return fail(ATTN_ERR_INVALID_ARG, "workspace too small: %zu bytes given, %zu needed", workspace_bytes, need);
  if (need > 0 && (st = check_ptr(workspace, "workspace"))) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == ATTN_BF16)
    return from_cuda(launch_bwd_bf16(pb, q, k, v, o, dout, lse, dq, dk, dv, workspace, s), "attn_bwd launch");
  return from_cuda(launch_bwd_fp32(pb, static_cast<const float*>(q), static_cast<const float*>(k),
                                   static_cast<const float*>(v), static_cast<const float*>(o),
                                   static_cast<const float*>(dout), lse, static_cast<float*>(dq),
                                   static_cast<float*>(dk), static_cast<float*>(dv), workspace, s),
                   "attn_bwd (fp32 check mode) launch");
}

attn_status attn_bwd_accumulate(const void* q, const void* k, const void* v, const void* o, const void* dout,
                                const float* lse, const int32_t* cu_seqlens, int32_t batch, int32_t seqlen,
                                int32_t max_seqlen, int32_t total_tokens, int32_t hq, int32_t hkv, int32_t d,
                                float scale, int32_t causal, float* dq_acc, float* dk_acc, float* dv_acc,
                                void* workspace, size_t workspace_bytes, void* stream) {
  Problem pb;
  attn_status st = (attn_status)bwd_check_args(q, k, v, o, dout, lse, cu_seqlens, batch, seqlen, max_seqlen,
                                               total_tokens, hq, hkv, d, scale, causal, ATTN_BF16, dq_acc, dk_acc,
                                               dv_acc, &pb);
  if (st != ATTN_OK) return st;
  if (total_tokens == 0 || batch == 0) return ok();
  const size_t need = attn_bwd_workspace_size(batch, pb.max_seqlen, total_tokens, hq, hkv, d, ATTN_BF16);
  if (workspace_bytes < need)
    return fail(ATTN_ERR_INVALID_ARG, "workspace too small: %zu bytes given, %zu needed", workspace_bytes, need);
  if ((st = check_ptr(workspace, "workspace"))) return st;
  return from_cuda(launch_bwd_bf16_accumulate(pb, q, k, v, o, dout, lse, dq_acc, dk_acc, dv_acc, workspace,
                                              static_cast<cudaStream_t>(stream)),
                   "attn_bwd_accumulate launch");
}

attn_status attn_get_device_error(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return from_cuda(e, "stream synchronize");
  uint32_t word = 0;
  const uint32_t zero = 0;
  e = cudaMemcpyFromSymbol(&word, g_device_error, sizeof word);
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof zero);
  if (e != cudaSuccess) return from_cuda(e, "reading the device error word");
  if (word & ATTN_DEVERR_TIMEOUT) return fail(ATTN_ERR_TIMEOUT, "a kernel's pipeline wait timed out");
  if (word & ATTN_DEVERR_SEQLEN) return fail(ATTN_ERR_INVALID_ARG, "a sequence is longer than max_seqlen");
  return ok();
}

attn_status attn_set_wait_limit_ns(uint64_t ns) {
  if (ns == 0) return fail(ATTN_ERR_INVALID_ARG, "the wait limit must be positive");
  const cudaError_t e = cudaMemcpyToSymbol(g_wait_limit_ns, &ns, sizeof ns);
  return from_cuda(e, "setting the wait limit");
}

uint64_t attn_get_wait_limit_ns(void) {
  uint64_t ns = 0;
  if (cudaMemcpyFromSymbol(&ns, g_wait_limit_ns, sizeof ns) != cudaSuccess) return 0;
  return ns;
}

attn_status attn_selftest_wait(int32_t arrive, void* stream) {
  if (arrive != 0 && arrive != 1) return fail(ATTN_ERR_INVALID_ARG, "arrive must be 0 or 1");
  return from_cuda(launch_selftest_wait(arrive, static_cast<cudaStream_t>(stream)), "selftest launch");
}

attn_status attn_selftest_exp2(const float* x, float* y_fma, float* y_sfu, int64_t n, void* stream) {
  if (n < 0) return fail(ATTN_ERR_INVALID_ARG, "negative element count");
  if (n == 0) return ok();
  if (x == nullptr || y_fma == nullptr || y_sfu == nullptr)
    return fail(ATTN_ERR_INVALID_ARG, "x, y_fma and y_sfu must be device pointers");
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(y_fma) | reinterpret_cast<uintptr_t>(y_sfu)) & 3u)
    return fail(ATTN_ERR_INVALID_ARG, "x, y_fma and y_sfu must be 4-byte aligned");
  return from_cuda(launch_selftest_exp2(x, y_fma, y_sfu, n, static_cast<cudaStream_t>(stream)), "selftest launch");
}

const char* attn_status_string(attn_status status) {
  switch (status) {
    case ATTN_OK: return "ok";
    case ATTN_ERR_INVALID_ARG: return "invalid argument";
    case ATTN_ERR_UNSUPPORTED: return "unsupported configuration";
    case ATTN_ERR_CUDA: return "CUDA error";
    case ATTN_ERR_TIMEOUT: return "device pipeline wait timed out";
  }
  return "unknown status";
}

const char* attn_last_error_message(void) { return g_last_error; }

attn_status attn_profile_enable(int32_t on) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_prof_on = on != 0;
  return ok();
}

int32_t attn_profile_kernel_count(void) { return K_NUM_KINDS; }

const char* attn_profile_kernel_name(int32_t kind) { return kernel_kind_name(kind); }

attn_status attn_profile_collect(double* total_ms, int64_t* launches, int32_t n) {
  std::vector<int> pending;
  {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    pending.swap(g_prof_pending);
  }
  attn_status st = ok();
  for (int idx : pending) {
    const EventPair& ep = g_prof_pool[idx];
    float ms = 0.f;
    cudaError_t e = cudaEventSynchronize(ep.end);
    if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, ep.start, ep.end);
    if (e != cudaSuccess) {
      st = from_cuda(e, "reading launch timing events");
    } else if (ep.kind < n) {
      if (total_ms) total_ms[ep.kind] += ms;
      if (launches) launches[ep.kind] += 1;
    }
  }
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (int idx : pending) g_prof_free.push_back(idx);
  return st;
}

int64_t attn_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int32_t attn_version(void) { return 100; }

}  // extern "C"
