// check_fp32.cu -- the fp32-input check mode: the same exact attention, forward and
// backward, in plain fp32 SIMT arithmetic (no tensor cores, accurate expf/logf).
//
// The tutorial "FlashAttention 与高效注意力内核" asks, in section 数值验证, that the
// forward agree with a float64 reference to a relative error of order 1e-5; fp32
// tensor-core modes cannot reach that, so this mode runs on the FMA pipes.  It keeps the
// method's structure -- K/V tiles staged in shared memory and the online softmax of
// section "Online Softmax 技巧" applied one key at a time (running max m, running sum l,
// rescaled running O) -- and writes only O and LSE = m + ln l.  The backward recomputes
// P_ij = exp(S_ij - LSE_i) from the saved statistic (section 反向) and applies
//   D_i = sum_c dO_ic O_ic, dS_ij = P_ij (dO_i . V_j - D_i),
//   dQ_i = scale sum_j dS_ij K_j,  dK_j = scale sum_i dS_ij Q_i,  dV_j = sum_i P_ij dO_i
// in two passes: one warp per query row for D and dQ, then one warp per key row for dK
// and dV (summed over the query heads of the GQA group), so nothing needs atomics.
#include <math.h>

#include "kernels.h"
#include "sm100.cuh"

namespace attn {

namespace {

constexpr int kRowsPerBlock = 8;   // one warp per row
constexpr int kChunk = 32;         // keys (or query rows) staged in shared memory at a time

struct SeqInfo {
  int start, len;
};

__device__ __forceinline__ SeqInfo seq_info(const int32_t* cu, int b, int seqlen) {
  SeqInfo s;
  s.start = cu ? cu[b] : b * seqlen;
  s.len = cu ? cu[b + 1] - s.start : seqlen;
  return s;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

template <int D>
__global__ void __launch_bounds__(256) fwd_fp32_kernel(const float* __restrict__ q, const float* __restrict__ k,
                                                       const float* __restrict__ v, Problem pb, float* __restrict__ o,
                                                       float* __restrict__ lse) {
  constexpr int E = D / 32;   // elements per lane
  __shared__ float sk[kChunk][D + 1];
  __shared__ float sv[kChunk][D + 1];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y, b = blockIdx.z;
  const int g = h / (pb.hq / pb.hkv);
  const SeqInfo si = seq_info(pb.cu_seqlens, b, pb.seqlen);
  if (si.len > pb.max_seqlen && threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.y == 0)
    report_error(ATTN_DEVERR_SEQLEN);
  const int r0 = blockIdx.x * kRowsPerBlock;
  if (r0 >= si.len) return;
  const int i = r0 + warp;
  const bool row_ok = i < si.len;
  const int last_row = min(si.len, r0 + kRowsPerBlock) - 1;
  const int nkeys = pb.causal ? last_row + 1 : si.len;

  float qv[E], acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    qv[e] = row_ok ? q[((size_t)(si.start + i) * pb.hq + h) * D + e * 32 + lane] : 0.f;
    acc[e] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  const int vis = row_ok ? (pb.causal ? i + 1 : si.len) : 0;
  for (int k0 = 0; k0 < nkeys; k0 += kChunk) {
    __syncthreads();
    for (int idx = threadIdx.x; idx < kChunk * D; idx += blockDim.x) {
      const int jj = idx / D, c = idx % D;
      const int j = k0 + jj;
      const bool in = j < si.len;
      sk[jj][c] = in ? k[((size_t)(si.start + j) * pb.hkv + g) * D + c] : 0.f;
      sv[jj][c] = in ? v[((size_t)(si.start + j) * pb.hkv + g) * D + c] : 0.f;
    }
    __syncthreads();
    const int jmax = min(kChunk, vis - k0);
    for (int jj = 0; jj < jmax; ++jj) {
      float part = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) part = fmaf(qv[e], sk[jj][e * 32 + lane], part);
      const float s = warp_sum(part) * pb.scale;
      const float m_new = fmaxf(m, s);
      const float corr = expf(m - m_new);
      const float pe = expf(s - m_new);
      l = l * corr + pe;
#pragma unroll
      for (int e = 0; e < E; ++e) acc[e] = fmaf(pe, sv[jj][e * 32 + lane], acc[e] * corr);
      m = m_new;
    }
  }
  if (row_ok) {
    const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) o[((size_t)(si.start + i) * pb.hq + h) * D + e * 32 + lane] = acc[e] * inv;
    if (lane == 0) lse[(size_t)h * pb.total_tokens + si.start + i] = l > 0.f ? m + logf(l) : -INFINITY;
  }
}

// Pass 1 of the backward: D_i and dQ_i, one warp per query row.
template <int D>
__global__ void __launch_bounds__(256) bwd_fp32_dq_kernel(const float* __restrict__ q, const float* __restrict__ k,
                                                          const float* __restrict__ v, const float* __restrict__ o,
                                                          const float* __restrict__ dout, const float* __restrict__ lse,
                                                          Problem pb, float* __restrict__ dq, float* __restrict__ dd) {
  constexpr int E = D / 32;
  __shared__ float sk[kChunk][D + 1];
  __shared__ float sv[kChunk][D + 1];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y, b = blockIdx.z;
  const int g = h / (pb.hq / pb.hkv);
  const SeqInfo si = seq_info(pb.cu_seqlens, b, pb.seqlen);
  if (si.len > pb.max_seqlen && threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.y == 0)
    report_error(ATTN_DEVERR_SEQLEN);
  const int r0 = blockIdx.x * kRowsPerBlock;
  if (r0 >= si.len) return;
  const int i = r0 + warp;
  const bool row_ok = i < si.len;
  const int last_row = min(si.len, r0 + kRowsPerBlock) - 1;
  const int nkeys = pb.causal ? last_row + 1 : si.len;
  const size_t qrow = ((size_t)(si.start + (row_ok ? i : 0)) * pb.hq + h) * D;

  float qv[E], dov[E], acc[E];
  float part = 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    qv[e] = row_ok ? q[qrow + e * 32 + lane] : 0.f;
    dov[e] = row_ok ? dout[qrow + e * 32 + lane] : 0.f;
    part = fmaf(dov[e], row_ok ? o[qrow + e * 32 + lane] : 0.f, part);
    acc[e] = 0.f;
  }
  const float Di = warp_sum(part);
  const float lse_i = row_ok ? lse[(size_t)h * pb.total_tokens + si.start + i] : 0.f;
  const int vis = row_ok ? (pb.causal ? i + 1 : si.len) : 0;
  for (int k0 = 0; k0 < nkeys; k0 += kChunk) {
    __syncthreads();
    for (int idx = threadIdx.x; idx < kChunk * D; idx += blockDim.x) {
      const int jj = idx / D, c = idx % D;
      const int j = k0 + jj;
      const bool in = j < si.len;
      sk[jj][c] = in ? k[((size_t)(si.start + j) * pb.hkv + g) * D + c] : 0.f;
      sv[jj][c] = in ? v[((size_t)(si.start + j) * pb.hkv + g) * D + c] : 0.f;
    }
    __syncthreads();
    const int jmax = min(kChunk, vis - k0);
    for (int jj = 0; jj < jmax; ++jj) {
      float ps = 0.f, pd = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        ps = fmaf(qv[e], sk[jj][e * 32 + lane], ps);
        pd = fmaf(dov[e], sv[jj][e * 32 + lane], pd);
      }
      const float s = warp_sum(ps) * pb.scale;
      const float dp = warp_sum(pd);
      const float pr = expf(s - lse_i);
      const float ds = pr * (dp - Di);
#pragma unroll
      for (int e = 0; e < E; ++e) acc[e] = fmaf(ds, sk[jj][e * 32 + lane], acc[e]);
    }
  }
  if (row_ok) {
#pragma unroll
    for (int e = 0; e < E; ++e) dq[qrow + e * 32 + lane] = acc[e] * pb.scale;
    if (lane == 0) dd[(size_t)h * pb.total_tokens + si.start + i] = Di;
  }
}

// Pass 2 of the backward: dK_j and dV_j, one warp per key row of one kv head, summed over
// the query heads of its group and over every query row that sees the key.
template <int D>
__global__ void __launch_bounds__(256) bwd_fp32_dkdv_kernel(const float* __restrict__ q, const float* __restrict__ k,
                                                            const float* __restrict__ v, const float* __restrict__ dout,
                                                            const float* __restrict__ lse, const float* __restrict__ dd,
                                                            Problem pb, float* __restrict__ dk, float* __restrict__ dv) {
  constexpr int E = D / 32;
  __shared__ float sq[kChunk][D + 1];
  __shared__ float sdo[kChunk][D + 1];
  __shared__ float slse[kChunk], sdd[kChunk];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.y, b = blockIdx.z;
  const int G = pb.hq / pb.hkv;
  const SeqInfo si = seq_info(pb.cu_seqlens, b, pb.seqlen);
  const int r0 = blockIdx.x * kRowsPerBlock;
  if (r0 >= si.len) return;
  const int j = r0 + warp;
  const bool key_ok = j < si.len;
  const size_t krow = ((size_t)(si.start + (key_ok ? j : 0)) * pb.hkv + g) * D;
  float kv_[E], vv[E], ak[E], av[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    kv_[e] = key_ok ? k[krow + e * 32 + lane] : 0.f;
    vv[e] = key_ok ? v[krow + e * 32 + lane] : 0.f;
    ak[e] = 0.f;
    av[e] = 0.f;
  }
  // causal: rows i >= j see key j; the block's smallest key bounds the first row needed
  const int row_begin = pb.causal ? r0 : 0;
  for (int hh = 0; hh < G; ++hh) {
    const int h = g * G + hh;
    for (int i0 = row_begin; i0 < si.len; i0 += kChunk) {
      __syncthreads();
      for (int idx = threadIdx.x; idx < kChunk * D; idx += blockDim.x) {
        const int ii = idx / D, c = idx % D;
        const int i = i0 + ii;
        const bool in = i < si.len;
        sq[ii][c] = in ? q[((size_t)(si.start + i) * pb.hq + h) * D + c] : 0.f;
        sdo[ii][c] = in ? dout[((size_t)(si.start + i) * pb.hq + h) * D + c] : 0.f;
      }
      if (threadIdx.x < kChunk) {
        const int i = i0 + threadIdx.x;
        const bool in = i < si.len;
        slse[threadIdx.x] = in ? lse[(size_t)h * pb.total_tokens + si.start + i] : 0.f;
        sdd[threadIdx.x] = in ? dd[(size_t)h * pb.total_tokens + si.start + i] : 0.f;
      }
      __syncthreads();
      if (!key_ok) continue;
      for (int ii = 0; ii < kChunk; ++ii) {
        const int i = i0 + ii;
        if (i >= si.len) break;
        if (pb.causal && i < j) continue;
        float ps = 0.f, pd = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) {
          ps = fmaf(sq[ii][e * 32 + lane], kv_[e], ps);
          pd = fmaf(sdo[ii][e * 32 + lane], vv[e], pd);
        }
        const float s = warp_sum(ps) * pb.scale;
        const float dp = warp_sum(pd);
        const float pr = expf(s - slse[ii]);
        const float ds = pr * (dp - sdd[ii]);
#pragma unroll
        for (int e = 0; e < E; ++e) {
          ak[e] = fmaf(ds, sq[ii][e * 32 + lane], ak[e]);
          av[e] = fmaf(pr, sdo[ii][e * 32 + lane], av[e]);
        }
      }
    }
  }
  if (key_ok) {
#pragma unroll
    for (int e = 0; e < E; ++e) {
      dk[krow + e * 32 + lane] = ak[e] * pb.scale;
      dv[krow + e * 32 + lane] = av[e];
    }
  }
}

template <int D>
cudaError_t fwd_fp32_d(const Problem& pb, const float* q, const float* k, const float* v, float* o, float* lse,
                       cudaStream_t st) {
  dim3 grid((pb.max_seqlen + kRowsPerBlock - 1) / kRowsPerBlock, pb.hq, pb.batch);
  LaunchScope scope(K_FWD_FP32, st);
  fwd_fp32_kernel<D><<<grid, 256, 0, st>>>(q, k, v, pb, o, lse);
  return cudaGetLastError();
}

template <int D>
cudaError_t bwd_fp32_d(const Problem& pb, const float* q, const float* k, const float* v, const float* o,
                       const float* dout, const float* lse, float* dq, float* dk, float* dv, float* dd,
                       cudaStream_t st) {
  dim3 g1((pb.max_seqlen + kRowsPerBlock - 1) / kRowsPerBlock, pb.hq, pb.batch);
  cudaError_t e;
  {
    LaunchScope scope(K_BWD_FP32_DQ, st);
    bwd_fp32_dq_kernel<D><<<g1, 256, 0, st>>>(q, k, v, o, dout, lse, pb, dq, dd);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) return e;
  dim3 g2((pb.max_seqlen + kRowsPerBlock - 1) / kRowsPerBlock, pb.hkv, pb.batch);
  LaunchScope scope(K_BWD_FP32_DKDV, st);
  bwd_fp32_dkdv_kernel<D><<<g2, 256, 0, st>>>(q, k, v, dout, lse, dd, pb, dk, dv);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_fp32(const Problem& pb, const float* q, const float* k, const float* v, float* o, float* lse,
                            cudaStream_t st) {
  if (pb.total_tokens == 0 || pb.batch == 0 || pb.max_seqlen == 0) return cudaSuccess;
  switch (pb.d) {
    case 32: return fwd_fp32_d<32>(pb, q, k, v, o, lse, st);
    case 64: return fwd_fp32_d<64>(pb, q, k, v, o, lse, st);
    case 128: return fwd_fp32_d<128>(pb, q, k, v, o, lse, st);
    default: return cudaErrorInvalidValue;
  }
}

size_t bwd_fp32_workspace_bytes(const Problem& pb) {
  return (size_t)pb.hq * (size_t)pb.total_tokens * sizeof(float);
}

cudaError_t launch_bwd_fp32(const Problem& pb, const float* q, const float* k, const float* v, const float* o,
                            const float* dout, const float* lse, float* dq, float* dk, float* dv, void* workspace,
                            cudaStream_t st) {
  if (pb.total_tokens == 0 || pb.batch == 0 || pb.max_seqlen == 0) return cudaSuccess;
  float* dd = static_cast<float*>(workspace);
  switch (pb.d) {
    case 32: return bwd_fp32_d<32>(pb, q, k, v, o, dout, lse, dq, dk, dv, dd, st);
    case 64: return bwd_fp32_d<64>(pb, q, k, v, o, dout, lse, dq, dk, dv, dd, st);
    case 128: return bwd_fp32_d<128>(pb, q, k, v, o, dout, lse, dq, dk, dv, dd, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace attn
