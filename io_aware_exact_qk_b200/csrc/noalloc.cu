// noalloc.cu -- attn_bwd_noalloc: the backward without a caller-provided workspace.
//
// Who needs this.  attn_bwd wants a workspace (the D statistics and the fp32 dQ
// accumulator) that the caller allocates.  Some callers cannot do that at the point
// where they run the backward: inference and training engines that reserve all of their
// device memory at start-up and forbid allocation afterwards (cudaMalloc can synchronise
// the device, stall, or fail once a caching allocator owns the free memory), and plain C
// hosts that link libattn.so directly and have no allocator of their own to hand a
// workspace from.  For them this entry point takes its scratch from a fixed array that
// lives in the library's own device globals, so nothing is allocated per call.
//
// How.  The scratch is the file-scope device array below, kNoAllocScratchBytes (64 MiB)
// long; every GPU on which the library is used holds it until the process exits.  In
// host code the array's name is only a host-side stand-in, not a device address, so the
// first call on each device looks its address up with cudaGetSymbolAddress (with that
// device current) and caches it; that first call should come before any stream capture.
// Every call shares the one array: the backward's preprocess kernel clears the dQ
// accumulator on every call, and calls whose work overlaps on the GPU (different streams,
// or different host threads on the same device) race on the scratch and must not be made.
#include <mutex>

#include "../../include/attn.h"
#include "kernels.h"

namespace attn {

namespace {

constexpr size_t kNoAllocScratchBytes = 64ull << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_setup_mu;
void* g_scratch_addr[kMaxDevices] = {nullptr};

// The device address of the scratch array on the current device (looked up once).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_setup_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace

}  // namespace attn

using namespace attn;

extern "C" attn_status attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                                        const void* dout, const float* lse, const int32_t* cu_seqlens,
                                        int32_t batch, int32_t seqlen, int32_t max_seqlen, int32_t total_tokens,
                                        int32_t hq, int32_t hkv, int32_t d, float scale, int32_t causal,
                                        int32_t dtype, void* dq, void* dk, void* dv, void* stream) {
  // Every argument is checked on the host first, exactly as attn_bwd checks them, so a
  // malformed call is refused before it touches the GPU (not even the scratch address is
  // looked up).
  Problem pb;
  const int st = bwd_check_args(q, k, v, o, dout, lse, cu_seqlens, batch, seqlen, max_seqlen, total_tokens, hq, hkv,
                                d, scale, causal, dtype, dq, dk, dv, &pb);
  if (st != ATTN_OK) return (attn_status)st;
  if (total_tokens == 0 || batch == 0) return ATTN_OK;
  const size_t need = attn_bwd_workspace_size(batch, pb.max_seqlen, total_tokens, hq, hkv, d, dtype);
  if (need > kNoAllocScratchBytes)
    return (attn_status)record_error(ATTN_ERR_INVALID_ARG,
                                     "attn_bwd_noalloc: this problem needs %zu bytes of scratch but the built-in "
                                     "scratch holds %zu (64 MiB); use attn_bwd with a workspace",
                                     need, kNoAllocScratchBytes);
  void* scratch = nullptr;
  if (need > 0) {
    const cudaError_t e = scratch_address(&scratch);
    if (e != cudaSuccess)
      return (attn_status)record_error(ATTN_ERR_CUDA, "attn_bwd_noalloc: looking up the scratch address: %s",
                                       cudaGetErrorString(e));
  }
  return attn_bwd(q, k, v, o, dout, lse, cu_seqlens, batch, seqlen, max_seqlen, total_tokens, hq, hkv, d, scale,
                  causal, dtype, dq, dk, dv, scratch, need, stream);
}
