// host_step.cu -- attn_fwd_bwd_host: one forward and one backward on HOST buffers, with the
// host <-> device copies overlapped with the kernels.
//
// Who needs this.  A caller whose Q, K, V and dO live in host memory (a CPU-side data
// pipeline, a C host without a device allocator of its own) would otherwise copy all
// inputs in, run attn_fwd and attn_bwd, and copy all results back, one after the other.
// The copies then dominate: at B = 4, H = 16, N = 4096, d = 128 each direction moves
// 268 MB over PCIe (~5 ms) against ~1.5 ms of kernels.
//
// How.  The sequences are cut into up to kMaxChunks groups of whole sequences with about
// equal token counts (attention never crosses a sequence boundary, so each group is an
// independent problem).  Three streams of the library's own, one per engine, run a
// pipeline over the groups: the copy-in stream uploads group c's rows of Q, K, V, dO (and
// its rebased cu_seqlens, all groups' at once); the compute stream, once they have arrived, runs attn_fwd and
// attn_bwd on that group alone; the copy-out stream then downloads its O, dQ, dK, dV rows
// and its block of LSE.  Uploads of later groups and downloads of earlier ones overlap the
// kernels, and the two copy directions overlap each other.  The call is ordered on the
// caller's stream like any other: its first copy waits for the work already queued there,
// and work queued there afterwards waits for its last copy.
//
// Device memory comes from the caller (attn_fwd_bwd_host_scratch_size bytes): full-size
// Q, K, V, dO, O, dQ, dK, dV, LSE, the groups' cu_seqlens, and one forward and one
// backward workspace that the groups use in turn on the compute stream.
#include <algorithm>
#include <mutex>
#include <vector>

#include "../../include/attn.h"
#include "kernels.h"

namespace attn {

namespace {

constexpr int kMaxChunks = 4;
constexpr int kMaxDevices = 64;

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Offsets of the device scratch regions (each 256-byte aligned).
struct HostLayout {
  size_t q, k, v, dout, o, dq, dk, dv, lse, cu, ws_fwd, ws_bwd, ws_bwd_bytes, total;
};

HostLayout host_layout(int32_t batch, int32_t total_tokens, int32_t hq, int32_t hkv, int32_t d) {
  HostLayout L{};
  const size_t T = (size_t)total_tokens;
  const size_t nq = T * hq * d * 2, nk = T * hkv * d * 2;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += align256(bytes);
    return at;
  };
  L.q = take(nq);
  L.k = take(nk);
  L.v = take(nk);
  L.dout = take(nq);
  L.o = take(nq);
  L.dq = take(nq);
  L.dk = take(nk);
  L.dv = take(nk);
  L.lse = take(T * hq * sizeof(float) + kMaxChunks * 256);   // each group's [hq, tokens] block 256-aligned
  L.cu = take(((size_t)batch + kMaxChunks + 1) * sizeof(int32_t));
  L.ws_fwd = take(attn_fwd_workspace_size(batch, total_tokens, total_tokens, hq, hkv, d, ATTN_BF16));
  // a group never has more tokens than the whole batch, so the full-size backward
  // workspace serves every group
  L.ws_bwd_bytes = attn_bwd_workspace_size(batch, total_tokens, total_tokens, hq, hkv, d, ATTN_BF16);
  L.ws_bwd = take(L.ws_bwd_bytes);
  L.total = off;
  return L;
}

// The library's three streams and the pipeline's events on one device.
struct Pipe {
  cudaStream_t in = nullptr, comp = nullptr, out = nullptr;
  cudaEvent_t start = nullptr, done = nullptr;
  cudaEvent_t arrived[kMaxChunks] = {}, computed[kMaxChunks] = {};
  std::mutex mu;   // one call at a time per device enqueues on these streams and events
};

std::mutex g_pipes_mu;
Pipe* g_pipes[kMaxDevices] = {nullptr};

cudaError_t pipe_for_current_device(Pipe** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_pipes_mu);
  if (g_pipes[dev] == nullptr) {
    Pipe* p = new Pipe();
    const unsigned ev = cudaEventDisableTiming;
    if ((e = cudaStreamCreateWithFlags(&p->in, cudaStreamNonBlocking)) != cudaSuccess ||
        (e = cudaStreamCreateWithFlags(&p->comp, cudaStreamNonBlocking)) != cudaSuccess ||
        (e = cudaStreamCreateWithFlags(&p->out, cudaStreamNonBlocking)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&p->start, ev)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&p->done, ev)) != cudaSuccess)
      return e;
    for (int c = 0; c < kMaxChunks; ++c)
      if ((e = cudaEventCreateWithFlags(&p->arrived[c], ev)) != cudaSuccess ||
          (e = cudaEventCreateWithFlags(&p->computed[c], ev)) != cudaSuccess)
        return e;
    g_pipes[dev] = p;
  }
  *out = g_pipes[dev];
  return cudaSuccess;
}

// One group of whole sequences: sequences [b0, b1), tokens [t0, t1).
struct Chunk {
  int b0, b1, t0, t1, max_len;
};

// Up to kMaxChunks groups with about equal token counts (each at least one sequence);
// empty groups are dropped.
std::vector<Chunk> make_chunks(const int32_t* cu, int32_t batch, int32_t seqlen) {
  auto start = [&](int b) { return cu ? cu[b] : b * seqlen; };
  const int total = start(batch);
  const int n = batch < kMaxChunks ? batch : kMaxChunks;
  std::vector<Chunk> out;
  int b = 0;
  for (int c = 0; c < n && b < batch; ++c) {
    const long long target = (long long)total * (c + 1) / n;
    Chunk ch{b, b, start(b), 0, 0};
    while (ch.b1 < batch && (ch.b1 == ch.b0 || start(ch.b1) < target || c == n - 1)) {
      ch.max_len = std::max(ch.max_len, start(ch.b1 + 1) - start(ch.b1));
      ++ch.b1;
    }
    ch.t1 = start(ch.b1);
    b = ch.b1;
    if (ch.t1 > ch.t0) out.push_back(ch);
  }
  return out;
}

}  // namespace

}  // namespace attn

using namespace attn;

extern "C" {

size_t attn_fwd_bwd_host_scratch_size(int32_t batch, int32_t total_tokens, int32_t hq, int32_t hkv, int32_t d) {
  if (batch < 0 || total_tokens <= 0 || hq <= 0 || hkv <= 0 || d <= 0) return 0;
  return host_layout(batch, total_tokens, hq, hkv, d).total;
}

attn_status attn_fwd_bwd_host(const void* q, const void* k, const void* v, const void* dout,
                              const int32_t* cu_seqlens, int32_t batch, int32_t seqlen, int32_t max_seqlen,
                              int32_t total_tokens, int32_t hq, int32_t hkv, int32_t d, float scale, int32_t causal,
                              void* o, float* lse, void* dq, void* dk, void* dv, void* scratch,
                              size_t scratch_bytes, void* stream) {
  // Host-side validation first: nothing is queued for a malformed call.  (The shape check
  // only tests cu_seqlens' alignment, so the host array can stand in for a device one.)
  Problem pb;
  attn_status st = (attn_status)validate_shapes(cu_seqlens, batch, seqlen, max_seqlen, total_tokens, hq, hkv, d,
                                                scale, causal, ATTN_BF16, &pb);
  if (st != ATTN_OK) return st;
  if (cu_seqlens != nullptr) {
    if (cu_seqlens[0] != 0 || cu_seqlens[batch] != total_tokens)
      return (attn_status)record_error(ATTN_ERR_INVALID_ARG, "cu_seqlens must start at 0 and end at total_tokens");
    for (int b = 0; b < batch; ++b) {
      const int len = cu_seqlens[b + 1] - cu_seqlens[b];
      if (len < 0)
        return (attn_status)record_error(ATTN_ERR_INVALID_ARG, "cu_seqlens decreases at sequence %d", b);
      if (len > max_seqlen)
        return (attn_status)record_error(ATTN_ERR_INVALID_ARG, "sequence %d is longer than max_seqlen", b);
    }
  }
  if (total_tokens == 0 || batch == 0) return (attn_status)status_ok();
  if (q == nullptr || k == nullptr || v == nullptr || dout == nullptr || o == nullptr || lse == nullptr ||
      dq == nullptr || dk == nullptr || dv == nullptr)
    return (attn_status)record_error(ATTN_ERR_INVALID_ARG, "a host tensor is NULL");
  const HostLayout L = host_layout(batch, total_tokens, hq, hkv, d);
  if (scratch_bytes < L.total)
    return (attn_status)record_error(ATTN_ERR_INVALID_ARG, "scratch too small: %zu bytes given, %zu needed",
                                     scratch_bytes, L.total);
  if ((st = (attn_status)validate_ptr(scratch, "scratch"))) return st;

  Pipe* pp = nullptr;
  cudaError_t e = pipe_for_current_device(&pp);
  if (e != cudaSuccess) return (attn_status)cuda_status(e, "attn_fwd_bwd_host setup");
  std::lock_guard<std::mutex> lk(pp->mu);
  const cudaStream_t caller = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(scratch);
  const size_t rq = (size_t)hq * d * 2, rk = (size_t)hkv * d * 2;   // bytes per token row
  auto dptr = [&](size_t region, size_t off) { return static_cast<void*>(base + region + off); };
  auto hptr = [](const void* h, size_t off) { return static_cast<const uint8_t*>(h) + off; };
  auto hout = [](void* h, size_t off) { return static_cast<void*>(static_cast<uint8_t*>(h) + off); };

  const std::vector<Chunk> chunks = make_chunks(cu_seqlens, batch, seqlen);
  // each group's LSE block [hq, tokens] at its own 256-byte aligned offset
  std::vector<size_t> lse_off(chunks.size());
  for (size_t c = 0, at = 0; c < chunks.size(); ++c) {
    lse_off[c] = at;
    at += align256((size_t)hq * (chunks[c].t1 - chunks[c].t0) * sizeof(float));
  }
  // the groups' cu_seqlens, rebased to their first token (group c's array at int offset b0 + c)
  std::vector<int32_t> cu_host;
  if (cu_seqlens != nullptr) {
    cu_host.assign((size_t)batch + kMaxChunks + 1, 0);
    for (size_t c = 0; c < chunks.size(); ++c)
      for (int b = chunks[c].b0; b <= chunks[c].b1; ++b) cu_host[b + c] = cu_seqlens[b] - chunks[c].t0;
  }

  attn_status result = ATTN_OK;
  auto check = [&](cudaError_t err, const char* what) {
    if (err != cudaSuccess && result == ATTN_OK) result = (attn_status)cuda_status(err, what);
    return err == cudaSuccess;
  };
  bool good = check(cudaEventRecord(pp->start, caller), "record start") &&
              check(cudaStreamWaitEvent(pp->in, pp->start, 0), "copy-in waits for the caller");
  // every group's cu_seqlens in one copy, ahead of the groups' rows (a small copy from
  // pageable memory, staged by the driver before the call returns)
  if (good && cu_seqlens != nullptr)
    good = check(cudaMemcpyAsync(dptr(L.cu, 0), cu_host.data(), cu_host.size() * sizeof(int32_t),
                                 cudaMemcpyHostToDevice, pp->in),
                 "copy cu_seqlens in");
  for (size_t c = 0; good && c < chunks.size(); ++c) {
    const Chunk& ch = chunks[c];
    const size_t t0 = (size_t)ch.t0, nt = (size_t)(ch.t1 - ch.t0);
    // copy-in: this group's rows of Q, K, V, dO
    good = check(cudaMemcpyAsync(dptr(L.q, t0 * rq), hptr(q, t0 * rq), nt * rq, cudaMemcpyHostToDevice, pp->in),
                 "copy Q in") &&
           check(cudaMemcpyAsync(dptr(L.k, t0 * rk), hptr(k, t0 * rk), nt * rk, cudaMemcpyHostToDevice, pp->in),
                 "copy K in") &&
           check(cudaMemcpyAsync(dptr(L.v, t0 * rk), hptr(v, t0 * rk), nt * rk, cudaMemcpyHostToDevice, pp->in),
                 "copy V in") &&
           check(cudaMemcpyAsync(dptr(L.dout, t0 * rq), hptr(dout, t0 * rq), nt * rq, cudaMemcpyHostToDevice,
                                 pp->in),
                 "copy dO in");
    int32_t* cu_dev =
        cu_seqlens ? static_cast<int32_t*>(dptr(L.cu, (size_t)(ch.b0 + c) * sizeof(int32_t))) : nullptr;
    good = good && check(cudaEventRecord(pp->arrived[c], pp->in), "record arrival") &&
           check(cudaStreamWaitEvent(pp->comp, pp->arrived[c], 0), "compute waits for the inputs");
    if (!good) break;
    // compute: forward and backward of this group alone; its LSE block is [hq, nt]
    const int nb = ch.b1 - ch.b0;
    const int sl = cu_seqlens ? 0 : seqlen;
    const int ms = cu_seqlens ? ch.max_len : seqlen;
    float* lse_c = reinterpret_cast<float*>(dptr(L.lse, lse_off[c]));
    attn_status s1 = attn_fwd(dptr(L.q, t0 * rq), dptr(L.k, t0 * rk), dptr(L.v, t0 * rk), cu_dev, nb, sl, ms,
                              (int)nt, hq, hkv, d, scale, causal, ATTN_BF16, dptr(L.o, t0 * rq), lse_c,
                              dptr(L.ws_fwd, 0), kFwdWorkspaceBytes, pp->comp);
    if (s1 == ATTN_OK)
      s1 = attn_bwd(dptr(L.q, t0 * rq), dptr(L.k, t0 * rk), dptr(L.v, t0 * rk), dptr(L.o, t0 * rq),
                    dptr(L.dout, t0 * rq), lse_c, cu_dev, nb, sl, ms, (int)nt, hq, hkv, d, scale, causal, ATTN_BF16,
                    dptr(L.dq, t0 * rq), dptr(L.dk, t0 * rk), dptr(L.dv, t0 * rk), dptr(L.ws_bwd, 0),
                    L.ws_bwd_bytes, pp->comp);
    if (s1 != ATTN_OK) {
      result = s1;
      break;
    }
    good = check(cudaEventRecord(pp->computed[c], pp->comp), "record compute") &&
           check(cudaStreamWaitEvent(pp->out, pp->computed[c], 0), "copy-out waits for the kernels");
    // copy-out: this group's rows of O, dQ, dK, dV and its LSE block (a 2-D copy into the
    // [hq, total_tokens] host layout)
    good = good &&
           check(cudaMemcpyAsync(hout(o, t0 * rq), dptr(L.o, t0 * rq), nt * rq, cudaMemcpyDeviceToHost, pp->out),
                 "copy O out") &&
           check(cudaMemcpyAsync(hout(dq, t0 * rq), dptr(L.dq, t0 * rq), nt * rq, cudaMemcpyDeviceToHost, pp->out),
                 "copy dQ out") &&
           check(cudaMemcpyAsync(hout(dk, t0 * rk), dptr(L.dk, t0 * rk), nt * rk, cudaMemcpyDeviceToHost, pp->out),
                 "copy dK out") &&
           check(cudaMemcpyAsync(hout(dv, t0 * rk), dptr(L.dv, t0 * rk), nt * rk, cudaMemcpyDeviceToHost, pp->out),
                 "copy dV out") &&
           check(cudaMemcpy2DAsync(lse + t0, (size_t)total_tokens * sizeof(float), lse_c, nt * sizeof(float),
                                   nt * sizeof(float), (size_t)hq, cudaMemcpyDeviceToHost, pp->out),
                 "copy LSE out");
  }
  if (good && result == ATTN_OK) {
    good = check(cudaEventRecord(pp->done, pp->out), "record done") &&
           check(cudaStreamWaitEvent(caller, pp->done, 0), "the caller waits for the copies");
    if (good) return (attn_status)status_ok();
  }
  // On a failure part of the pipeline may be queued: let it finish before returning, so
  // that no copy is still writing into the caller's buffers afterwards.
  cudaStreamSynchronize(pp->in);
  cudaStreamSynchronize(pp->comp);
  cudaStreamSynchronize(pp->out);
  return result;
}

}  // extern "C"
