// kernels.h -- internal launch interface between the C ABI layer and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace attn {

// One attention problem as described by the C ABI's shape arguments.
struct Problem {
  const int32_t* cu_seqlens;  // device prefix sums [batch + 1], or nullptr for batch mode
  int32_t batch;              // number of sequences
  int32_t seqlen;             // batch mode: tokens per sequence
  int32_t max_seqlen;         // >= every sequence length
  int32_t total_tokens;       // T
  int32_t hq, hkv, d;
  float scale;
  int32_t causal;
};

// Forward, bf16 tensors (tcgen05 path).  o [T,hq,d] bf16, lse [hq,T] f32; workspace:
// kFwdWorkspaceBytes (the work-item counter).
constexpr size_t kFwdWorkspaceBytes = 256;
cudaError_t launch_fwd_bf16(const Problem& pb, const void* q, const void* k, const void* v, void* o,
                            float* lse, void* workspace, cudaStream_t stream);

// Backward, bf16 tensors (tcgen05 path).  Workspace: bwd_bf16_workspace_bytes(pb).
size_t bwd_bf16_workspace_bytes(const Problem& pb);
cudaError_t launch_bwd_bf16(const Problem& pb, const void* q, const void* k, const void* v, const void* o,
                            const void* dout, const float* lse, void* dq, void* dk, void* dv, void* workspace,
                            cudaStream_t stream);

// The same backward adding its gradients into the caller's float32 dq_acc [T,hq,d],
// dk_acc and dv_acc [T,hkv,d] (read-add-write; nothing bf16 is written).  Workspace:
// bwd_bf16_workspace_bytes(pb) (its dQ accumulator part goes unused).
cudaError_t launch_bwd_bf16_accumulate(const Problem& pb, const void* q, const void* k, const void* v, const void* o,
                                       const void* dout, const float* lse, float* dq_acc, float* dk_acc,
                                       float* dv_acc, void* workspace, cudaStream_t stream);

// Decoding-shaped forward (split-KV): sequence b has Lq query rows (the newest positions)
// and Lk keys.  q [Tq,hq,d], k/v [Tk,hkv,d], o [Tq,hq,d] bf16, lse [hq,Tq] f32.
struct DecodeProblem {
  const int32_t* cu_q;   // device prefix sums [batch + 1], or nullptr (fixed seqlen_q)
  const int32_t* cu_k;   // device prefix sums [batch + 1], or nullptr (fixed seqlen_k)
  int32_t batch, seqlen_q, seqlen_k, max_seqlen_q, max_seqlen_k, total_q, total_k;
  int32_t hq, hkv, d;
  float scale;
  int32_t causal;
  int32_t num_splits;    // requested key splits, 0 = chosen from the shape and the SM count
  int32_t varlen;        // lengths come from cu_q / cu_k (only their bounds are known on the host)
};
struct DecodeSplit {
  int tiles_per_split, n_splits;
  size_t o_part_bytes, workspace_bytes;
};
DecodeSplit decode_split(const DecodeProblem& pb);
cudaError_t launch_decode_bf16(const DecodeProblem& pb, const void* q, const void* k, const void* v, void* o,
                               float* lse, void* workspace, cudaStream_t stream);

// Merge of partial results over disjoint key sets (ring attention): o_acc [T,hq,d] f32,
// lse_acc [hq,T] f32 accumulate bf16 partials o_part [T,hq,d] / lse_part [hq,T].
cudaError_t launch_merge_partial(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part,
                                 int total_tokens, int hq, int d, int first, cudaStream_t stream);
cudaError_t launch_merge_finish(const float* o_acc, void* o, int total_tokens, int hq, int d, cudaStream_t stream);

// FP8 forward (d = 64 or 128; fixed-length batches or cu_seqlens): e4m3 Q8, K8 [tokens,
// heads, d] and V^T [batch * hkv][d][fp8_vt_pitch(max_seqlen)] with per-head descales;
// bf16 O, fp32 LSE.
inline int fp8_vt_pitch(int seqlen) { return (seqlen + 15) / 16 * 16; }
cudaError_t launch_fwd_fp8(const Problem& pb, const void* q8, const void* k8, const void* vt8,
                           const float* descale_q, const float* descale_k, const float* descale_v, void* o,
                           float* lse, void* workspace, cudaStream_t stream);
// Per-head e4m3 quantisation of bf16 Q, K, V into those operands (cu_seqlens nullptr:
// batch sequences of seqlen tokens; else packed sequences of at most max_seqlen tokens).
cudaError_t launch_fp8_quantize(const void* q, const void* k, const void* v, const int32_t* cu_seqlens, int batch,
                                int seqlen, int max_seqlen, int total_tokens, int hq, int hkv, int d, void* q8,
                                void* k8, void* vt8, float* descale_q, float* descale_k, float* descale_v,
                                cudaStream_t stream);

// fp32 check mode (SIMT fp32 arithmetic).
cudaError_t launch_fwd_fp32(const Problem& pb, const float* q, const float* k, const float* v, float* o,
                            float* lse, cudaStream_t stream);
size_t bwd_fp32_workspace_bytes(const Problem& pb);
cudaError_t launch_bwd_fp32(const Problem& pb, const float* q, const float* k, const float* v, const float* o,
                            const float* dout, const float* lse, float* dq, float* dk, float* dv, void* workspace,
                            cudaStream_t stream);

// Diagnostics (diag.cu): a bounded wait that completes (arrive != 0) or runs out, and
// the forward's FMA-pipe 2^x next to the special-function unit's, element by element.
cudaError_t launch_selftest_wait(int arrive, cudaStream_t stream);
cudaError_t launch_selftest_exp2(const float* x, float* y_fma, float* y_sfu, int64_t n, cudaStream_t stream);

// Launch bookkeeping: every kernel launch is wrapped in a LaunchScope, which counts it
// and, while timing is enabled, brackets it with CUDA events on its stream.
enum KernelKind : int {
  K_FWD_BF16 = 0,
  K_BWD_PREPROCESS,
  K_BWD_BF16,
  K_BWD_DQ_CONVERT,
  K_FWD_FP32,
  K_BWD_FP32_DQ,
  K_BWD_FP32_DKDV,
  K_DECODE_BF16,
  K_DECODE_COMBINE,
  K_MERGE_PARTIAL,
  K_MERGE_FINISH,
  K_FWD_FP8,
  K_FP8_QUANTIZE,
  K_SELFTEST,
  K_NUM_KINDS
};
const char* kernel_kind_name(int kind);
struct LaunchScope {
  LaunchScope(int kind, cudaStream_t stream);
  ~LaunchScope();
  int kind;
  cudaStream_t stream;
  int slot;   // event pair index, -1 when timing is off
};

// Host validation of attn_bwd's arguments (everything but the workspace); returns an
// attn_status value and, on failure, records the reason.  Touches no GPU state.
int bwd_check_args(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                   const int32_t* cu_seqlens, int32_t batch, int32_t seqlen, int32_t max_seqlen,
                   int32_t total_tokens, int32_t hq, int32_t hkv, int32_t d, float scale, int32_t causal,
                   int32_t dtype, void* dq, void* dk, void* dv, Problem* pb);

// Records `fmt` as the calling thread's last error message (attn_last_error_message) and
// returns `status`.
int record_error(int status, const char* fmt, ...);
// The entry points' shared host checks, for entry points in other files (each returns an
// attn_status value and, on failure, records the reason): shape arguments (fills `pb`), a
// device pointer (non-NULL, 16-byte aligned), a CUDA result, and success (clears the
// message).
int validate_shapes(const int32_t* cu_seqlens, int32_t batch, int32_t seqlen, int32_t max_seqlen, int32_t total_tokens,
                    int32_t hq, int32_t hkv, int32_t d, float scale, int32_t causal, int32_t dtype, Problem* pb);
int validate_ptr(const void* p, const char* name);
int cuda_status(cudaError_t e, const char* what);
int status_ok();

// Host helper shared by the launchers: encodes a 3-D bf16 TMA descriptor over a
// [rows, heads, d] tensor with a (box_inner x 1 x box_rows) box and the swizzle that
// matches a box_inner * 2-byte row (128 B or 64 B).
bool encode_tma_3d(void* tmap_out, const void* base, int d, int heads, int rows, int box_inner, int box_rows);
// The same with a box spanning `box_heads` consecutive heads (box_inner x box_heads x
// box_rows); the tile lands in shared memory as rows (token, head), head fastest.
bool encode_tma_3d_box(void* tmap_out, const void* base, int d, int heads, int rows, int box_inner, int box_heads,
                       int box_rows);
// A 3-D tensor of bytes (e4m3) with extents dim0 (contiguous) x dim1 x dim2, the byte
// strides of dims 1 and 2, and a box0 x box1 x box2 box; a 128- or 64-byte box row uses
// the swizzle of that span.
bool encode_tma_u8_3d(void* tmap_out, const void* base, int dim0, int dim1, int dim2, uint64_t stride1,
                      uint64_t stride2, int box0, int box1, int box2);
// The same over an fp32 [rows, heads, d] tensor; a 32-float (128-byte) box row uses the
// 128-byte swizzle, any other width is unswizzled.  Used for bulk reductions.
bool encode_tma_3d_f32(void* tmap_out, const void* base, int d, int heads, int rows, int box_inner, int box_rows);

}  // namespace attn
