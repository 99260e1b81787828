// diag.cu -- self-test kernels behind the library's diagnostic entry points.
//
//   selftest_wait    one CTA waits on an mbarrier with the bounded wait every pipeline in
//                    the library uses.  With `arrive` the barrier's phase completes and
//                    the wait returns at once; without it nothing ever arrives, so the wait
//                    runs out after the device's wait limit and records
//                    ATTN_DEVERR_TIMEOUT.  This is how the timeout path is exercised on a
//                    GPU without breaking a real pipeline: the kernel holds no TMA copy,
//                    MMA or TMEM allocation that would still be in flight when it gives up.
//   selftest_exp2    evaluates, for each input, the forward kernel's FMA-pipe 2^x
//                    (ex2_fma_pair) and the special-function unit's ex2.approx, so that a
//                    test can hold the former to its stated error bound.
#include <algorithm>

#include "kernels.h"
#include "sm100.cuh"

namespace attn {

namespace {

__global__ void __launch_bounds__(32) selftest_wait_kernel(int arrive) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) {
    if (arrive) mbar_arrive(smem_u32(&bar));
    mbar_wait(smem_u32(&bar), 0, &abort_flag);   // phase 0 completes on the single arrival
  }
}

__global__ void __launch_bounds__(256) selftest_exp2_kernel(const float* __restrict__ x, float* __restrict__ y_fma,
                                                            float* __restrict__ y_sfu, int64_t n) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; 2 * i < n; i += stride) {
    const float x0 = x[2 * i];
    const float x1 = 2 * i + 1 < n ? x[2 * i + 1] : x0;
    float p0, p1;
    ex2_fma_pair(f2(x0, x1), p0, p1);
    y_fma[2 * i] = p0;
    y_sfu[2 * i] = ex2(x0);
    if (2 * i + 1 < n) {
      y_fma[2 * i + 1] = p1;
      y_sfu[2 * i + 1] = ex2(x1);
    }
  }
}

}  // namespace

cudaError_t launch_selftest_wait(int arrive, cudaStream_t stream) {
  LaunchScope scope(K_SELFTEST, stream);
  selftest_wait_kernel<<<1, 32, 0, stream>>>(arrive);
  return cudaGetLastError();
}

cudaError_t launch_selftest_exp2(const float* x, float* y_fma, float* y_sfu, int64_t n, cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  const int64_t pairs = (n + 1) / 2;
  const int blocks = (int)std::min<int64_t>((pairs + 255) / 256, 4096);
  LaunchScope scope(K_SELFTEST, stream);
  selftest_exp2_kernel<<<blocks, 256, 0, stream>>>(x, y_fma, y_sfu, n);
  return cudaGetLastError();
}

}  // namespace attn
