/*
 * attn.h -- C ABI of libattn.so: exact scaled-dot-product attention, forward and
 * backward, on one NVIDIA B200 (sm_100a).
 *
 * The operation (the "FlashAttention 与高效注意力内核：IO 感知与分块计算" tutorial,
 * section 标准注意力三步, with the 1/sqrt(d)-style scale of the "Flash-Attention" concept
 * page, section 核心思想):
 *
 *     S = scale * Q K^T   (S_ij = -inf where causal and key j > query i)
 *     P = softmax(S)      row by row
 *     O = P V
 *
 * computed IO-aware: Q/K/V tiles are staged in on-chip memory, the softmax is the
 * online (running max m, running sum l, rescaled running O) form of the tutorial's
 * section "Online Softmax 技巧", and only O and the per-row statistic
 * LSE_i = m_i + ln l_i (natural log, in units of the scaled scores) reach HBM (section
 * "前向").  The backward recomputes S and P from Q, K, V and LSE (section "反向") and
 * applies D_i = sum_c dO_ic O_ic, dP = dO V^T, dS = P o (dP - D),
 * dQ = scale dS K, dK = scale dS^T Q, dV = P^T dO.
 *
 * Grouped-query attention ("相关工作" page, paper 6): query head h reads K/V head
 * h / (hq / hkv).  Variable-length packing (the tutorial's 验证清单, 变长序列打包):
 * sequences are concatenated on the token axis and described by cu_seqlens; attention
 * never crosses a sequence boundary; a zero-length sequence is legal and writes nothing.
 * Causal masking is top-left aligned inside each sequence: query i sees keys j <= i.
 *
 * ---- Conventions shared by every entry point ----------------------------------------
 *
 * Layouts (row-major, innermost dimension contiguous, no padding):
 *     q, o, dout, dq   [total_tokens, hq,  d]
 *     k, v, dk, dv     [total_tokens, hkv, d]
 *     lse              [hq, total_tokens]            float32
 * Element type: ATTN_BF16 -- q/k/v/o/dout/dq/dk/dv are bfloat16, statistics and all
 * accumulation are float32; ATTN_FP32 -- the fp32-input check mode, every tensor is
 * float32 (computed with float32 arithmetic throughout; slow, for numerical checks).
 *
 * Shapes: batch mode passes cu_seqlens = NULL, `batch` sequences of `seqlen` tokens,
 * total_tokens = batch * seqlen.  Varlen mode passes cu_seqlens, a DEVICE int32 array of
 * batch + 1 prefix sums with cu_seqlens[0] = 0 and cu_seqlens[batch] = total_tokens;
 * `seqlen` is ignored and `max_seqlen` must be >= every sequence length (a sequence
 * longer than max_seqlen is reported by attn_get_device_error as ATTN_ERR_INVALID_ARG).
 * Supported: d in {32, 64, 128}; hq % hkv == 0; scale > 0 and finite.
 *
 * Pointers are DEVICE pointers into memory the caller owns; every tensor pointer must
 * be 16-byte aligned.  The library never allocates or frees memory; scratch space is the
 * caller's `workspace` (size from the *_workspace_size queries; it may be NULL when the
 * size is 0).  `stream` is a cudaStream_t (NULL = the legacy default stream); every
 * call only enqueues work on it and returns without synchronising.
 *
 * Errors: arguments are validated on the host before anything is launched, so an
 * ATTN_ERR_INVALID_ARG / ATTN_ERR_UNSUPPORTED return leaves every output untouched;
 * attn_last_error_message() then says which argument was wrong.  A failed launch returns
 * ATTN_ERR_CUDA.  Kernels never trap: a device-side problem (a pipeline wait that timed
 * out, a sequence longer than max_seqlen) sets a per-device error word that
 * attn_get_device_error() reads and clears.
 */
#ifndef ATTN_H
#define ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    ATTN_OK = 0,
    ATTN_ERR_INVALID_ARG = 1,   /* a pointer, size or shape argument is invalid          */
    ATTN_ERR_UNSUPPORTED = 2,   /* valid but outside what this library supports (d, dtype) */
    ATTN_ERR_CUDA = 3,          /* a CUDA runtime or driver call failed                  */
    ATTN_ERR_TIMEOUT = 4        /* a kernel's bounded pipeline wait ran out              */
} attn_status;

typedef enum {
    ATTN_BF16 = 0,              /* bf16 tensors, fp32 accumulation (the fast path)       */
    ATTN_FP32 = 1               /* fp32 tensors, fp32 arithmetic (numerical check mode)  */
} attn_dtype;

/* Forward.  Writes o [T,hq,d] and lse [hq,T].
 * Defined by: tutorial sections 标准注意力三步 (the result), 分块 / Online Softmax 技巧
 * (how it is reached) and 前向 (only O and the row statistics are stored).
 * Workspace (bf16 mode): attn_fwd_workspace_size() = 256 bytes, the counter from which the
 * persistent kernel's CTAs claim work items; it is reset on the stream before each launch,
 * so calls that overlap (other streams) need workspaces of their own. */
attn_status attn_fwd(const void *q, const void *k, const void *v,
                     const int32_t *cu_seqlens, int32_t batch, int32_t seqlen,
                     int32_t max_seqlen, int32_t total_tokens,
                     int32_t hq, int32_t hkv, int32_t d,
                     float scale, int32_t causal, int32_t dtype,
                     void *o, float *lse,
                     void *workspace, size_t workspace_bytes, void *stream);

/* Backward.  Reads q, k, v, the forward's o and lse, and the upstream gradient dout;
 * writes dq [T,hq,d], dk and dv [T,hkv,d] (dk/dv summed over each GQA group).
 * Defined by: tutorial sections 反向 and 反向重算流程 (recompute S and P per tile from
 * Q/K/V and the saved statistics, then form dQ/dK/dV from dO).
 * Workspace (bf16 mode): D [hq,T] float32 and a float32 dQ accumulator [T,hq,d]. */
attn_status attn_bwd(const void *q, const void *k, const void *v,
                     const void *o, const void *dout, const float *lse,
                     const int32_t *cu_seqlens, int32_t batch, int32_t seqlen,
                     int32_t max_seqlen, int32_t total_tokens,
                     int32_t hq, int32_t hkv, int32_t d,
                     float scale, int32_t causal, int32_t dtype,
                     void *dq, void *dk, void *dv,
                     void *workspace, size_t workspace_bytes, void *stream);

/* Backward into float32 accumulators: the gradients of the same backward (bf16 q, k, v,
 * o, dout; float32 lse; same shape arguments and causal rule as attn_bwd) are ADDED to
 *     dq_acc [T,hq,d],  dk_acc and dv_acc [T,hkv,d]      float32, DEVICE, 16-byte aligned
 * (read-add-write; they must hold the running sums, zero before the first call) and nothing
 * is written in bf16.  For computations that sum gradients over several calls -- ring
 * attention's backward sums one call per K/V block it visits ("相关工作" page, paper 7) --
 * this keeps the sum in float32 instead of rounding every call's gradients to bf16.  A
 * call's contributions equal attn_bwd's before their bf16 rounding (dK, dQ include the
 * scale).  Workspace: attn_bwd_workspace_size(..., ATTN_BF16).  Errors as attn_bwd; calls
 * that add into the same accumulators must not overlap on the GPU. */
attn_status attn_bwd_accumulate(const void *q, const void *k, const void *v,
                                const void *o, const void *dout, const float *lse,
                                const int32_t *cu_seqlens, int32_t batch, int32_t seqlen,
                                int32_t max_seqlen, int32_t total_tokens,
                                int32_t hq, int32_t hkv, int32_t d,
                                float scale, int32_t causal,
                                float *dq_acc, float *dk_acc, float *dv_acc,
                                void *workspace, size_t workspace_bytes, void *stream);

/* Backward without a caller-provided workspace.  (The pages describe no counterpart; this
 * exists for callers that cannot allocate device memory where they run the backward:
 * engines that reserve all device memory up front and forbid allocation later, and plain
 * C hosts with no allocator to take a workspace from.)  Same arguments, layouts and
 * results as attn_bwd, minus the workspace: the scratch comes from a 64 MiB array in the
 * library's device globals, held on every GPU that uses the library until the process
 * exits.  A problem whose attn_bwd_workspace_size() exceeds 64 MiB is rejected with
 * ATTN_ERR_INVALID_ARG (attn_last_error_message() says how much it needs); nothing is ever
 * allocated.  The first call on each device looks up the array's device address (with
 * that device current); make that first call before any stream capture.  Every call
 * shares the one array, and the backward clears the parts that must start at zero on
 * every call; calls whose GPU work overlaps (other streams, other host threads on the
 * same device) race on it and must not be made. */
attn_status attn_bwd_noalloc(const void *q, const void *k, const void *v,
                             const void *o, const void *dout, const float *lse,
                             const int32_t *cu_seqlens, int32_t batch, int32_t seqlen,
                             int32_t max_seqlen, int32_t total_tokens,
                             int32_t hq, int32_t hkv, int32_t d,
                             float scale, int32_t causal, int32_t dtype,
                             void *dq, void *dk, void *dv, void *stream);

/* One forward and one backward on HOST buffers, with the host <-> device copies overlapped
 * with the kernels: attn_fwd then attn_bwd (the tutorial's 前向 and 反向重算流程) for callers
 * whose tensors live in host memory.
 *   q, k, v, dout (inputs) and o, lse, dq, dk, dv (outputs): HOST arrays in the layouts of
 *       attn_fwd / attn_bwd (bf16; lse float32 [hq, total_tokens]); they should be
 *       page-locked (cudaHostAlloc / cudaHostRegister), or the copies overlap nothing;
 *   cu_seqlens: NULL (batch sequences of seqlen tokens) or a HOST int32 array [batch + 1]
 *       starting at 0, ending at total_tokens, never decreasing, no step above max_seqlen;
 *   scratch: caller-owned DEVICE memory of attn_fwd_bwd_host_scratch_size() bytes, 16-byte
 *       aligned (the device copies of all tensors, the groups' cu_seqlens, and one forward
 *       and one backward workspace).
 * The sequences are split into up to four groups of whole sequences with about equal token
 * counts; on three streams of the library's own, each group's rows are copied in, its
 * forward and backward run, and its results are copied out while the other groups copy.
 * Results are those of attn_fwd / attn_bwd on each group (O, LSE, dK, dV bit-identical to a
 * single call on all sequences; dQ up to the order of its fp32 sums).  Ordering: the first
 * copy waits for the work queued on `stream` before the call, and work queued on `stream`
 * afterwards waits for the last copy; the host outputs are complete once `stream` is
 * synchronised; calls that share a scratch must be ordered (one stream, or events), as calls
 * on one stream are.  Enqueueing is serialised per device.  Errors: those of attn_fwd / attn_bwd
 * and ATTN_ERR_INVALID_ARG for a malformed cu_seqlens, a NULL host array or a small or
 * unaligned scratch, all found on the host before anything is queued; a failing CUDA call
 * returns ATTN_ERR_CUDA after the part of the pipeline already queued has finished. */
size_t attn_fwd_bwd_host_scratch_size(int32_t batch, int32_t total_tokens,
                                      int32_t hq, int32_t hkv, int32_t d);
attn_status attn_fwd_bwd_host(const void *q, const void *k, const void *v, const void *dout,
                              const int32_t *cu_seqlens, int32_t batch, int32_t seqlen,
                              int32_t max_seqlen, int32_t total_tokens,
                              int32_t hq, int32_t hkv, int32_t d, float scale, int32_t causal,
                              void *o, float *lse, void *dq, void *dk, void *dv,
                              void *scratch, size_t scratch_bytes, void *stream);

/* Decoding forward (split-KV).  The tutorial's FlashDecoding variant (section
 * "FlashAttention 变体族谱": one query against a long KV, the KV cut into blocks whose
 * partial results are computed in parallel and then reduced; section "变体选择场景":
 * decoding is bandwidth-bound).  The result is the forward's definition for sequences whose
 * query rows are the newest positions of a longer key/value sequence: sequence b has
 * Lq_b query rows and Lk_b keys, and under `causal` query row t (0-based) sees keys
 * j <= Lk_b - Lq_b + t (bottom-right alignment; with Lq_b = Lk_b this is attn_fwd's mask).
 *     q, o   [total_q, hq, d]  bf16        k, v  [total_k, hkv, d]  bf16
 *     lse    [hq, total_q]     float32 (natural log; -inf and O = 0 for a row with no key)
 * Shapes: batch mode passes cu_seqlens_q = cu_seqlens_k = NULL and fixed seqlen_q /
 * seqlen_k (total_q = batch * seqlen_q, total_k = batch * seqlen_k); varlen mode passes
 * both DEVICE prefix-sum arrays (int32[batch + 1]) and bounds max_seqlen_q / max_seqlen_k
 * (a sequence exceeding them is reported by attn_get_device_error as
 * ATTN_ERR_INVALID_ARG).  The hq / hkv query heads of a KV head and their newest
 * max_seqlen_q tokens share one 128-row tile: (hq / hkv) * max_seqlen_q <= 128, else
 * ATTN_ERR_UNSUPPORTED.  d in {32, 64, 128}; bf16 only.
 * num_splits: key splits per (sequence, KV head); 0 lets the library choose from the
 * shape and the SM count.  With more than one split the partial results go through the
 * caller's workspace (attn_fwd_decode_workspace_size() bytes, same num_splits) and a
 * combine kernel; with one split the workspace is unused (may be NULL, size 0). */
attn_status attn_fwd_decode(const void *q, const void *k, const void *v,
                            const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                            int32_t batch, int32_t seqlen_q, int32_t seqlen_k,
                            int32_t max_seqlen_q, int32_t max_seqlen_k,
                            int32_t total_q, int32_t total_k,
                            int32_t hq, int32_t hkv, int32_t d,
                            float scale, int32_t causal, int32_t num_splits,
                            void *o, float *lse,
                            void *workspace, size_t workspace_bytes, void *stream);

/* Workspace bytes attn_fwd_decode needs (0 when one split suffices) for the same shape
 * arguments; varlen = 1 when cu_seqlens_q / cu_seqlens_k will be passed (batch mode: the
 * max_seqlen values are seqlen_q / seqlen_k).  With num_splits == 0 the split count, and so
 * the size, depends on the current device's SM count: query it on the device that runs
 * the call. */
size_t attn_fwd_decode_workspace_size(int32_t batch, int32_t max_seqlen_q, int32_t max_seqlen_k,
                                      int32_t total_q, int32_t total_k, int32_t hq, int32_t hkv,
                                      int32_t d, int32_t varlen, int32_t num_splits);

/* Merge of partial results over disjoint key sets, the building block of ring attention
 * ("相关工作" page, paper 7: each device attends its queries to the K/V block it holds,
 * and the blocks travel around a ring).  For one row, partials (O_a, LSE_a) and
 * (O_b, LSE_b) over disjoint keys combine exactly as the tutorial's section 修正公式
 * combines blocks:  LSE = ln(e^LSE_a + e^LSE_b),  O = e^(LSE_a - LSE) O_a + e^(LSE_b - LSE) O_b.
 * attn_merge_partial folds a bf16 partial (o_part [T,hq,d], lse_part [hq,T], e.g. one
 * attn_fwd result) into the float32 accumulators o_acc [T,hq,d] and lse_acc [hq,T];
 * first = 1 starts them from that partial (their contents are ignored).  A partial row
 * with LSE = -inf (no visible key) contributes nothing.  attn_merge_finish writes
 * o = bf16(o_acc) [T,hq,d].  d in {32, 64, 128}; device pointers, 16-byte aligned. */
attn_status attn_merge_partial(float *o_acc, float *lse_acc, const void *o_part, const float *lse_part,
                               int32_t total_tokens, int32_t hq, int32_t d, int32_t first, void *stream);
attn_status attn_merge_finish(const float *o_acc, void *o, int32_t total_tokens, int32_t hq, int32_t d,
                              void *stream);

/* FP8 (e4m3) forward operands.  The "Flash-Attention" concept page names FP8 attention
 * (FlashAttention-3 on H100, 观察 2) and quantised attention with scaling (设计空间, 路线 4);
 * the scaling chosen here is one factor per head and tensor.
 * Reads bf16 q [batch*seqlen, hq, d], k and v [batch*seqlen, hkv, d] (a fixed-length
 * batch; d = 64 or 128; attn_fp8_quantize_varlen below takes packed sequences) and writes, all on the device, caller-allocated, 16-byte aligned:
 *   descale_q [hq], descale_k [hkv], descale_v [hkv] float32: amax over the head / 448
 *       (1 for an all-zero head), 448 being the largest finite e4m3 value;
 *   q8 [batch*seqlen, hq, d], k8 [batch*seqlen, hkv, d] bytes: e4m3 of x / descale
 *       (fp32 division, round to nearest even, saturating);
 *   vt8 [batch*hkv][d][pitch] bytes, pitch = seqlen rounded up to a multiple of 16:
 *       the same for v, transposed per (sequence, kv head) so that tokens are contiguous;
 *       the padding columns are zero.
 * Errors: ATTN_ERR_UNSUPPORTED for d other than 64 or 128; ATTN_ERR_INVALID_ARG for NULL
 * or unaligned pointers and negative sizes.  Asynchronous on `stream`. */
attn_status attn_fp8_quantize(const void *q, const void *k, const void *v,
                              int32_t batch, int32_t seqlen, int32_t hq, int32_t hkv, int32_t d,
                              void *q8, void *k8, void *vt8,
                              float *descale_q, float *descale_k, float *descale_v, void *stream);

/* FP8 forward: O = softmax(scale * (dq Q8)(dk K8)^T [+ causal mask]) (dv V8), per head
 * (the tutorial's 标准注意力三步 on the dequantised operands, reached by the same online
 * softmax as attn_fwd, with both products on e4m3 tensor cores).  Inputs are what
 * attn_fp8_quantize writes (same layouts, same fixed-length batch, d = 64 or 128).  The
 * probabilities that multiply V are rounded to e4m3 without a scale: the running row
 * maximum only moves when a tile's maximum exceeds it by more than 8 (log2 units), so every
 * probability lies in [0, 256], inside e4m3's range.  The row sums use the unrounded
 * probabilities.  Writes o [batch*seqlen, hq, d] bf16 and lse [hq, batch*seqlen] float32
 * (of the dequantised scores).  Workspace: attn_fwd_workspace_size(..., ATTN_BF16) = 256
 * bytes, as for attn_fwd.  Errors as attn_fwd; d other than 64 or 128 is
 * ATTN_ERR_UNSUPPORTED. */
attn_status attn_fwd_fp8(const void *q8, const void *k8, const void *vt8,
                         const float *descale_q, const float *descale_k, const float *descale_v,
                         int32_t batch, int32_t seqlen, int32_t hq, int32_t hkv, int32_t d,
                         float scale, int32_t causal, void *o, float *lse,
                         void *workspace, size_t workspace_bytes, void *stream);

/* The two FP8 calls over packed sequences of different lengths (the variable-length layout
 * of attn_fwd): sequence b holds tokens cu_seqlens[b] .. cu_seqlens[b+1] - 1 of q, k, v, q8,
 * k8, o (cu_seqlens: batch + 1 int32 on the device, non-decreasing, cu_seqlens[0] = 0,
 * cu_seqlens[batch] = total_tokens; no sequence longer than max_seqlen).  V^T is
 * vt8 [batch*hkv][d][pitch] with pitch = max_seqlen rounded up to a multiple of 16, sequence
 * b's tokens in columns 0 .. len_b - 1 and zeros after them; the descales are per head over
 * all sequences, as in the fixed-length calls.  attn_fwd_fp8_varlen reads what
 * attn_fp8_quantize_varlen wrote with the same cu_seqlens and max_seqlen.  A sequence
 * longer than max_seqlen is reported by attn_get_device_error (ATTN_ERR_INVALID_ARG); its
 * V^T is cut at the pitch.  Errors: as the fixed-length calls, and ATTN_ERR_INVALID_ARG for
 * a NULL cu_seqlens or max_seqlen > total_tokens. */
attn_status attn_fp8_quantize_varlen(const void *q, const void *k, const void *v,
                                     const int32_t *cu_seqlens, int32_t batch, int32_t max_seqlen,
                                     int32_t total_tokens, int32_t hq, int32_t hkv, int32_t d,
                                     void *q8, void *k8, void *vt8,
                                     float *descale_q, float *descale_k, float *descale_v,
                                     void *stream);
attn_status attn_fwd_fp8_varlen(const void *q8, const void *k8, const void *vt8,
                                const float *descale_q, const float *descale_k,
                                const float *descale_v, const int32_t *cu_seqlens, int32_t batch,
                                int32_t max_seqlen, int32_t total_tokens, int32_t hq, int32_t hkv,
                                int32_t d, float scale, int32_t causal, void *o, float *lse,
                                void *workspace, size_t workspace_bytes, void *stream);

/* Workspace bytes attn_fwd / attn_bwd need for these shape arguments (0 = none). */
size_t attn_fwd_workspace_size(int32_t batch, int32_t max_seqlen, int32_t total_tokens,
                               int32_t hq, int32_t hkv, int32_t d, int32_t dtype);
size_t attn_bwd_workspace_size(int32_t batch, int32_t max_seqlen, int32_t total_tokens,
                               int32_t hq, int32_t hkv, int32_t d, int32_t dtype);

/* Synchronises `stream`, then reads and clears the current device's error word.
 * Returns ATTN_OK, ATTN_ERR_TIMEOUT, ATTN_ERR_INVALID_ARG (max_seqlen too small) or
 * ATTN_ERR_CUDA (the synchronisation itself failed). */
attn_status attn_get_device_error(void *stream);

/* Static description of a status code. */
const char *attn_status_string(attn_status status);

/* Human-readable reason for the last non-OK return on the calling thread ("" if none). */
const char *attn_last_error_message(void);

/* ---- launch timing (tracing) ----------------------------------------------------------
 * Off by default.  While enabled, every kernel the library launches is bracketed by a
 * pair of CUDA events recorded on the launch's stream.  attn_profile_collect()
 * synchronises those events, adds each launch's duration (milliseconds) and count into
 * total_ms[kind] / launches[kind] for kind < n, and forgets them.  Kinds are numbered
 * 0 .. attn_profile_kernel_count() - 1 and named by attn_profile_kernel_name().
 * attn_launch_count() counts every kernel launch since the library was loaded, enabled
 * or not.  The event pool is owned by the library; nothing is allocated on the device. */
attn_status attn_profile_enable(int32_t on);
int32_t attn_profile_kernel_count(void);
const char *attn_profile_kernel_name(int32_t kind);
attn_status attn_profile_collect(double *total_ms, int64_t *launches, int32_t n);
int64_t attn_launch_count(void);

/* ---- failure detection and self-tests -------------------------------------------------
 * Every pipeline wait inside the library's kernels is bounded in wall time.  A wait that
 * runs out marks its CTA aborted (the CTA's other roles stop waiting), records a timeout in
 * the device error word and lets the kernel return, so a broken pipeline ends as
 * ATTN_ERR_TIMEOUT from attn_get_device_error() instead of a hung GPU.  (The pages define no
 * such mechanism; it is this library's failure detection.)
 *
 * attn_set_wait_limit_ns sets the bound for the CURRENT device, in nanoseconds (default
 * 2 000 000 000, 2 s; 0 is ATTN_ERR_INVALID_ARG); attn_get_wait_limit_ns reads it (0 if the
 * read failed).  It is a per-device global that kernels read while they wait: change it
 * between calls, not while the library's kernels run.  A limit far below a kernel's normal
 * waits (a few microseconds) turns ordinary waits into timeouts.
 *
 * attn_selftest_wait launches one CTA that waits on a barrier with that same bounded wait.
 * arrive = 1: the barrier completes and the wait returns at once.  arrive = 0: nothing
 * arrives, the wait runs out after the limit and attn_get_device_error() reports
 * ATTN_ERR_TIMEOUT; the CTA holds no copy, MMA or Tensor Memory when it gives up, and the
 * GPU stays usable.  Asynchronous on `stream`.
 *
 * attn_selftest_exp2 writes, for n floats x (device pointers, 4-byte aligned), y_fma[i] =
 * the forward kernel's FMA-pipe evaluation of 2^x[i] and y_sfu[i] = the special-function
 * unit's approximate 2^x[i], so that the former can be checked against its error bound
 * (relative error below 7.6e-5 for x in [-125, 8]; 7.51e-5 at worst).  Asynchronous on `stream`. */
attn_status attn_set_wait_limit_ns(uint64_t ns);
uint64_t attn_get_wait_limit_ns(void);
attn_status attn_selftest_wait(int32_t arrive, void *stream);
attn_status attn_selftest_exp2(const float *x, float *y_fma, float *y_sfu, int64_t n, void *stream);

/* Library version, major * 10000 + minor * 100 + patch. */
int32_t attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_H */
