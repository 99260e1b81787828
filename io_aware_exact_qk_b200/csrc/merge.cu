// merge.cu -- merging partial attention results computed over disjoint key sets.
//
// When the keys of a row are split into disjoint sets (the devices of ring attention,
// "相关工作" page, paper 7 "Ring Attention with Blockwise Transformers": each device's
// local attention covers the K/V block it currently holds), each set s gives a partial
// result (O_s = its softmax-weighted values, LSE_s = ln of its sum of exponentials).  The
// exact result over the union is the online-softmax correction of the "FlashAttention 与
// 高效注意力内核" tutorial (section 修正公式) applied to whole sets:
//     LSE = ln(exp(LSE_a) + exp(LSE_b)),   O = exp(LSE_a - LSE) O_a + exp(LSE_b - LSE) O_b.
// attn_merge_partial folds one bf16 partial into a float32 accumulator (O_acc, LSE_acc);
// attn_merge_finish rounds the accumulated O to bf16.  A set with no visible key has
// LSE_s = -inf and contributes nothing; a row without any key stays O = 0, LSE = -inf.
#include <algorithm>

#include "kernels.h"
#include "sm100.cuh"

namespace attn {

namespace {

constexpr float kLog2e = 1.4426950408889634f;

// One warp per (token, head) row; D / 32 elements per lane.
template <int D>
__global__ void __launch_bounds__(256) merge_partial_kernel(float* __restrict__ o_acc, float* __restrict__ lse_acc,
                                                            const __nv_bfloat16* __restrict__ o_part,
                                                            const float* __restrict__ lse_part, int total_tokens,
                                                            int hq, int first) {
  constexpr int PER_LANE = D / 32;
  const int lane = threadIdx.x & 31;
  const int64_t rows = (int64_t)total_tokens * hq;
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t rw = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); rw < rows; rw += nwarps) {
    const int tok = (int)(rw / hq), h = (int)(rw % hq);
    const size_t li = (size_t)h * total_tokens + tok;
    float* acc = o_acc + (size_t)rw * D + lane * PER_LANE;
    const __nv_bfloat16* part = o_part + (size_t)rw * D + lane * PER_LANE;
    const float lp = lse_part[li];
    const float la = first ? -INFINITY : lse_acc[li];
    const float m = fmaxf(la, lp);
    float wa = 0.f, wp = 0.f, lse = -INFINITY;
    if (m != -INFINITY) {
      wa = la == -INFINITY ? 0.f : exp2f((la - m) * kLog2e);
      wp = lp == -INFINITY ? 0.f : exp2f((lp - m) * kLog2e);
      const float s = wa + wp;
      wa /= s;
      wp /= s;
      lse = m + logf(s);
    }
#pragma unroll
    for (int e = 0; e < PER_LANE; ++e) {
      const float a = first ? 0.f : acc[e];
      acc[e] = wa * a + wp * __bfloat162float(part[e]);
    }
    __syncwarp();   // every lane has read lse_acc before lane 0 overwrites it
    if (lane == 0) lse_acc[li] = lse;
  }
}

__global__ void __launch_bounds__(256) merge_finish_kernel(const float* __restrict__ o_acc, __nv_bfloat16* __restrict__ o,
                                                           int64_t n8) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += (int64_t)gridDim.x * blockDim.x) {
    const float4 a = reinterpret_cast<const float4*>(o_acc)[2 * i];
    const float4 b = reinterpret_cast<const float4*>(o_acc)[2 * i + 1];
    reinterpret_cast<uint4*>(o)[i] = make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(b.x, b.y),
                                                pack_bf16x2(b.z, b.w));
  }
}

int merge_sm_count() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  }
  return n;
}

}  // namespace

cudaError_t launch_merge_partial(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part,
                                 int total_tokens, int hq, int d, int first, cudaStream_t stream) {
  const int64_t rows = (int64_t)total_tokens * hq;
  if (rows == 0) return cudaSuccess;
  const int blocks = (int)std::min<int64_t>((rows + 7) / 8, (int64_t)merge_sm_count() * 16);
  const __nv_bfloat16* part = static_cast<const __nv_bfloat16*>(o_part);
  LaunchScope scope(K_MERGE_PARTIAL, stream);
  switch (d) {
    case 32: merge_partial_kernel<32><<<blocks, 256, 0, stream>>>(o_acc, lse_acc, part, lse_part, total_tokens, hq, first); break;
    case 64: merge_partial_kernel<64><<<blocks, 256, 0, stream>>>(o_acc, lse_acc, part, lse_part, total_tokens, hq, first); break;
    case 128: merge_partial_kernel<128><<<blocks, 256, 0, stream>>>(o_acc, lse_acc, part, lse_part, total_tokens, hq, first); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_merge_finish(const float* o_acc, void* o, int total_tokens, int hq, int d, cudaStream_t stream) {
  const int64_t n8 = (int64_t)total_tokens * hq * d / 8;
  if (n8 == 0) return cudaSuccess;
  const int blocks = (int)std::min<int64_t>((n8 + 255) / 256, (int64_t)merge_sm_count() * 16);
  LaunchScope scope(K_MERGE_FINISH, stream);
  merge_finish_kernel<<<blocks, 256, 0, stream>>>(o_acc, static_cast<__nv_bfloat16*>(o), n8);
  return cudaGetLastError();
}

}  // namespace attn
