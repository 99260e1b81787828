// decode_sm100.cu -- split-KV decoding forward for sm_100a (bf16): TMA + tcgen05 + TMEM.
//
// What it computes: the forward of exact attention for decoding-shaped problems, where a
// sequence has few query rows (the newest tokens) and a long key/value cache.  Sequence b
// has Lq query rows and Lk keys; the query rows are the LAST Lq positions, so under the
// causal mask row t sees keys j <= Lk - Lq + t.  Result: O [Tq, hq, d] bf16 and
// LSE [hq, Tq] fp32, the same definition as the forward (S = scale Q K^T, P = softmax(S),
// O = P V; LSE = m + ln l).
//
// How: the "FlashAttention 与高效注意力内核" tutorial's FlashDecoding entry (section
// "FlashAttention 变体族谱"): the key/value sequence is cut into splits that different CTAs
// process in parallel, each producing a partial result, and a reduce step combines them
// (section "变体选择场景": decoding is bandwidth-bound, so parallelism has to come from the
// key axis).  Per split the CTA runs the online softmax of section "Online Softmax 技巧"
// over its 128-key tiles and writes its partial O_s (already divided by its own row sum
// l_s) and LSE_s; the combine kernel then forms, per row,
//     LSE = ln sum_s exp(LSE_s),   O = sum_s exp(LSE_s - LSE) O_s,
// which is exactly the softmax over the union of the splits (the tutorial's 修正公式 applied
// to whole splits).  With a single split the CTA writes O and LSE directly.
//
// Query rows of one KV head's G query heads are packed into one 128-row tile (row
// r = t * G + hh for token t, head hh of the group), so the K/V tiles each CTA streams are
// read once for all G heads: the tensor core computes S = Q K^T over a 128-row tile of
// which only G * Lq rows are real (decode is HBM-bound; the padded MMA work is far below
// the memory time of the same tile).
//
// Roles (192 threads): warps 0-3 softmax + epilogue (one query row per thread; warps with
// no real row stay idle), warp 4 TMA producer, warp 5 MMA issuer.  TMEM: S double buffer at
// columns [0,128) and [128,256), O at [256, 256 + d).  Per key tile i: S(i) = Q K_i^T into
// buffer i % 2; softmax writes P(i) (bf16) over it; PV(i) accumulates O; S(i+2) reuses the
// buffer after PV(i) (tensor-core order).
#include <algorithm>

#include "kernels.h"
#include "sm100.cuh"

namespace attn {

namespace {

constexpr int kRows = 128;                 // query rows per tile == TMEM lanes
constexpr int kKeys = 128;                 // keys per K/V tile
constexpr float kRescaleSkip = 8.0f;       // log2 units: the running max moves only past this
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kThreads = 192;
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;

template <int D>
struct DecCfg {
  static constexpr int SW = D >= 64 ? 128 : 64;    // swizzle span == SMEM row pitch (bytes)
  static constexpr int PANEL = SW / 2;             // bf16 elements per panel row
  static constexpr int NPANEL = D / PANEL;
  static constexpr int PANEL_BYTES = kRows * SW;   // one panel of a 128-row tile
  static constexpr int TILE_BYTES = kRows * D * 2;
  static constexpr int STAGES = D == 128 ? 3 : 4;  // K/V ring depth (3 x 64 KB in flight at d = 128)
  static constexpr uint32_t SWZ = SW == 128 ? 2u : 4u;
  static constexpr int SBO = 8 * SW;
  static constexpr int KSTEPS_PER_PANEL = SW / 32;
  static constexpr int B_QFULL = 0;
  static constexpr int B_KFULL = 1;                  // STAGES
  static constexpr int B_VFULL = B_KFULL + STAGES;
  static constexpr int B_KEMPTY = B_VFULL + STAGES;
  static constexpr int B_VEMPTY = B_KEMPTY + STAGES;
  static constexpr int B_SFULL = B_VEMPTY + STAGES;  // 2 (one per S buffer)
  static constexpr int B_PFULL = B_SFULL + 2;        // arrived once per active softmax warp
  static constexpr int B_PVDONE = B_PFULL + 1;       // committed after every PV
  static constexpr int B_DRAIN = B_PVDONE + 1;       // the MMA issuer's completion at exit
  static constexpr int NBARS = B_DRAIN + 1;
  static constexpr int DATA_BYTES = (1 + 2 * STAGES) * TILE_BYTES;
  static constexpr int SMEM_BYTES = 1024 + DATA_BYTES + NBARS * 8 + 16;
};

struct DecParams {
  const int32_t* cu_q;     // device prefix sums [batch + 1] or nullptr (fixed seqlen_q)
  const int32_t* cu_k;     // device prefix sums [batch + 1] or nullptr (fixed seqlen_k)
  int32_t seqlen_q, seqlen_k, max_seqlen_q, max_seqlen_k, total_q, total_k;
  int32_t hq, hkv, G;
  int32_t tiles_per_split, n_splits;
  float scale_log2;        // scale * log2(e) in fp32
  double lse_skew;         // scale_log2 * ln 2 - scale (the rounding of scale_log2)
  int32_t causal;
  __nv_bfloat16* o;        // [Tq, hq, d]  (written directly when n_splits == 1)
  float* lse;              // [hq, Tq]
  float* o_part;           // [n_splits, Tq, hq, d] fp32, each split's O_s = its O / its l
  float* lse_part;         // [n_splits, hq, Tq]
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    decode_bf16_sm100(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const DecParams p) {
  using C = DecCfg<D>;
  const int sp = blockIdx.x;   // split
  const int g = blockIdx.y;    // kv head
  const int b = blockIdx.z;    // sequence
  const int q0 = p.cu_q ? p.cu_q[b] : b * p.seqlen_q;
  const int lq = p.cu_q ? p.cu_q[b + 1] - q0 : p.seqlen_q;
  const int k0 = p.cu_k ? p.cu_k[b] : b * p.seqlen_k;
  const int lk = p.cu_k ? p.cu_k[b + 1] - k0 : p.seqlen_k;
  if (lq > p.max_seqlen_q || lk > p.max_seqlen_k) {   // the tile box / split grid would not cover it
    if (threadIdx.x == 0) report_error(ATTN_DEVERR_SEQLEN);
    return;
  }
  const int R = p.G * lq;                  // packed query rows, <= 128
  const int j0 = sp * p.tiles_per_split;   // first key tile of this split
  const int n = max(0, min((lk + kKeys - 1) / kKeys, j0 + p.tiles_per_split) - j0);
  if (R == 0) return;
  if (n == 0) {
    // No key in this split: the combine skips a split whose LSE is -inf.  Unsplit (a
    // sequence with no keys), write the defined result of a row with no visible key.
    for (int r = threadIdx.x; r < R; r += blockDim.x) {
      const int tok = q0 + r / p.G, h = g * p.G + r % p.G;
      if (p.n_splits > 1) {
        p.lse_part[((size_t)sp * p.hq + h) * p.total_q + tok] = -INFINITY;
      } else {
        p.lse[(size_t)h * p.total_q + tok] = -INFINITY;
        uint4* dst = reinterpret_cast<uint4*>(p.o + ((size_t)tok * p.hq + h) * D);
        for (int e = 0; e < D / 8; ++e) dst[e] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    return;
  }

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  const uint32_t sQ = smem_u32(smem);
  const uint32_t sK = sQ + C::TILE_BYTES;
  const uint32_t sV = sK + C::STAGES * C::TILE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::DATA_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NBARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto bar = [&](int i) { return smem_u32(bars + i); };
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_active = (R + 31) / 32;      // softmax warps holding at least one real row

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NBARS; ++i) mbar_init(bar(i), i == C::B_PFULL ? (uint32_t)n_active : 1u);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  if (warp == kProducerWarp && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kProducerWarp) {
    // ---------------- TMA producer: the packed Q tile once, then the split's K/V tiles ----
    if (lane == 0) {
      // The Q box is (panel, G heads, max_seqlen_q tokens): rows t * G + hh of the tile.
      mbar_arrive_expect_tx(bar(C::B_QFULL), (uint32_t)(D * 2 * p.G * p.max_seqlen_q));
      for (int pn = 0; pn < C::NPANEL; ++pn)
        tma_load_3d(sQ + pn * C::PANEL_BYTES, &tmQ, bar(C::B_QFULL), pn * C::PANEL, g * p.G, q0);
      int kc = 0, vc = 0;   // K and V loads issued
      for (int i = 0; i < n; ++i) {
        const int s = i % C::STAGES;
        const uint32_t ph = (i / C::STAGES) & 1;
        const int key = k0 + (j0 + i) * kKeys;
        if (!mbar_wait(bar(C::B_KEMPTY + s), ph ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(bar(C::B_KFULL + s), C::TILE_BYTES);
        for (int pn = 0; pn < C::NPANEL; ++pn)
          tma_load_3d(sK + s * C::TILE_BYTES + pn * C::PANEL_BYTES, &tmK, bar(C::B_KFULL + s), pn * C::PANEL, g, key);
        ++kc;
        if (!mbar_wait(bar(C::B_VEMPTY + s), ph ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(bar(C::B_VFULL + s), C::TILE_BYTES);
        for (int pn = 0; pn < C::NPANEL; ++pn)
          tma_load_3d(sV + s * C::TILE_BYTES + pn * C::PANEL_BYTES, &tmV, bar(C::B_VFULL + s), pn * C::PANEL, g, key);
        ++vc;
      }
      // Every load issued here lands before the CTA releases its memory, also when another
      // role gave up waiting: only the last load of each stage can still be in flight.
      mbar_wait_drain(bar(C::B_QFULL), 0);
      for (int i = kc > C::STAGES ? kc - C::STAGES : 0; i < kc; ++i)
        mbar_wait_drain(bar(C::B_KFULL + i % C::STAGES), (i / C::STAGES) & 1);
      for (int i = vc > C::STAGES ? vc - C::STAGES : 0; i < vc; ++i)
        mbar_wait_drain(bar(C::B_VFULL + i % C::STAGES), (i / C::STAGES) & 1);
    }
  } else if (warp == kMmaWarp) {
    // ---------------- MMA issuer: S(0), S(1), then PV(i), S(i+2) ----------------
    if (lane == 0) {
      const uint32_t idesc_qk = idesc_bf16_f32(kRows, kKeys, false, false);
      const uint32_t idesc_pv = idesc_bf16_f32(kRows, D, false, true);
      const uint64_t q_desc = smem_desc(sQ, 16, C::SBO, C::SWZ);
      const uint64_t k_desc = smem_desc(sK, 16, C::SBO, C::SWZ);
      const uint64_t v_desc = smem_desc(sV, C::PANEL_BYTES, C::SBO, C::SWZ);
      auto issue_s = [&](int i) {
        const int s = i % C::STAGES;
        if (!mbar_wait(bar(C::B_KFULL + s), (i / C::STAGES) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(i & 1) * kKeys;
        const uint64_t b0 = desc_advance(k_desc, (uint32_t)s * C::TILE_BYTES);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / C::KSTEPS_PER_PANEL) * C::PANEL_BYTES + (kk % C::KSTEPS_PER_PANEL) * 32;
          mma_ss(d_tmem, desc_advance(q_desc, off), desc_advance(b0, off), idesc_qk, kk > 0 ? 1u : 0u);
        }
        mma_commit(bar(C::B_SFULL + (i & 1)));
        mma_commit(bar(C::B_KEMPTY + s));
        return true;
      };
      bool ok = mbar_wait(bar(C::B_QFULL), 0, abort_flag) && issue_s(0) && (n < 2 || issue_s(1));
      for (int i = 0; ok && i < n; ++i) {
        const int s = i % C::STAGES;
        if (!mbar_wait(bar(C::B_PFULL), i & 1, abort_flag)) break;
        if (!mbar_wait(bar(C::B_VFULL + s), (i / C::STAGES) & 1, abort_flag)) break;
        tc_fence_after();
        const uint64_t b0 = desc_advance(v_desc, (uint32_t)s * C::TILE_BYTES);
#pragma unroll
        for (int kk = 0; kk < kKeys / 16; ++kk)
          mma_ts(tmem + 2 * kKeys, tmem + (uint32_t)(i & 1) * kKeys + kk * 8, desc_advance(b0, kk * 16 * C::SW),
                 idesc_pv, (i > 0 || kk > 0) ? 1u : 0u);
        mma_commit(bar(C::B_VEMPTY + s));
        mma_commit(bar(C::B_PVDONE));
        if (i + 2 < n) ok = issue_s(i + 2);
      }
      // every MMA issued here has completed before the CTA frees Tensor Memory
      mma_commit(bar(C::B_DRAIN));
      mbar_wait_drain(bar(C::B_DRAIN), 0);
    }
  } else if (warp < n_active) {
    // ---------------- softmax + epilogue, one packed query row per thread ----------------
    const int lane_base = warp * 32;
    const int row = lane_base + lane;
    const bool row_ok = row < R;
    const int t = row / p.G;                      // token inside the sequence
    const int h = g * p.G + row % p.G;            // query head
    const int qpos = lk - lq + t;                 // the row's position among the keys
    const uint32_t trow = tmem + ((uint32_t)lane_base << 16);
    const float sl2 = p.scale_log2;
    float m_used = -INFINITY, mx_used = 0.f, l = 0.f;
    bool ok = true;
    for (int i = 0; i < n; ++i) {
      const uint32_t tS = trow + (uint32_t)(i & 1) * kKeys;
      if (!mbar_wait(bar(C::B_SFULL + (i & 1)), (i >> 1) & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      float s[kKeys];
      {
        uint32_t r0[32], r1[32], r2[32], r3[32];
        tmem_ld32(tS + 0, r0);
        tmem_ld32(tS + 32, r1);
        tmem_ld32(tS + 64, r2);
        tmem_ld32(tS + 96, r3);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          s[c] = __uint_as_float(r0[c]);
          s[32 + c] = __uint_as_float(r1[c]);
          s[64 + c] = __uint_as_float(r2[c]);
          s[96 + c] = __uint_as_float(r3[c]);
        }
      }
      // key kbase + c is visible iff it is in the sequence and, when causal, not after the row
      const int kbase = (j0 + i) * kKeys;
      int lim = lk - 1 - kbase;
      if (p.causal) lim = min(lim, qpos - kbase);
      if (lim < kKeys - 1) {
#pragma unroll
        for (int c = 0; c < kKeys; ++c)
          if (c > lim) s[c] = -INFINITY;
      }
      float mp[8];
#pragma unroll
      for (int a = 0; a < 8; ++a) mp[a] = fmaxf(s[a], s[8 + a]);
#pragma unroll
      for (int c = 16; c < kKeys; c += 16)
#pragma unroll
        for (int a = 0; a < 8; ++a) mp[a] = max3(mp[a], s[c + a], s[c + 8 + a]);
      const float mx = max3(max3(mp[0], mp[1], mp[2]), max3(mp[3], mp[4], mp[5]), fmaxf(mp[6], mp[7]));
      const float m_cand = mx * sl2;
      float m_new = m_used;
      if (m_cand > m_used + kRescaleSkip) {
        m_new = m_cand;
        mx_used = mx;
      }
      const float m_sub = (m_new == -INFINITY) ? 0.f : m_new;
      const uint64_t sl2x2 = f2(sl2, sl2);
      const uint64_t negm = f2(-m_sub, -m_sub);
      uint64_t sum2[4] = {f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f)};
      uint32_t pk[64];
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        float x0, x1;
        f2_split(fma2(f2(s[2 * c], s[2 * c + 1]), sl2x2, negm), x0, x1);
        const float p0 = ex2(x0), p1 = ex2(x1);
        sum2[c & 3] = add2(sum2[c & 3], f2(p0, p1));
        pk[c] = pack_bf16x2(p0, p1);
      }
      float sum_lo, sum_hi;
      f2_split(add2(add2(sum2[0], sum2[1]), add2(sum2[2], sum2[3])), sum_lo, sum_hi);
      const float rowsum = sum_lo + sum_hi;
      {
        uint32_t (&lo)[32] = *reinterpret_cast<uint32_t(*)[32]>(&pk[0]);
        uint32_t (&hi)[32] = *reinterpret_cast<uint32_t(*)[32]>(&pk[32]);
        tmem_st32(tS + 0, lo);
        tmem_st32(tS + 32, hi);
      }
      float alpha = 1.f;
      if (m_new != m_used) {
        alpha = ex2(m_used - m_sub);   // 0 when m_used is -inf
        l = l * alpha + rowsum;
      } else {
        l += rowsum;
      }
      const bool need = (i > 0) && (m_new != m_used);
      m_used = m_new;
      if (i > 0) {
        // O holds PV(i-1)'s sum once that product is done (waited every step, so each
        // phase of the barrier is observed in order).
        if (!mbar_wait(bar(C::B_PVDONE), (i - 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
      }
      if (__any_sync(0xffffffffu, need)) {
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(trow + 2 * kKeys + c * 32, r);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
          tmem_st32(trow + 2 * kKeys + c * 32, r);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::B_PFULL));
    }
    // ---------------- epilogue: this split's O / l and LSE ----------------
    if (ok && mbar_wait(bar(C::B_PVDONE), (n - 1) & 1, abort_flag)) {
      tc_fence_after();
      uint32_t r[D / 32][32];
#pragma unroll
      for (int c = 0; c < D / 32; ++c) tmem_ld32(trow + 2 * kKeys + c * 32, r[c]);
      tmem_wait_ld();
      if (row_ok) {
        const int tok = q0 + t;
        const float inv_l = l > 0.f ? 1.f / l : 0.f;
        // LSE = m ln 2 + ln l in double from the exact fp32 values used, minus the
        // first-order effect of scale_log2 being rounded to fp32.
        float lse = -INFINITY;
        if (l > 0.f)
          lse = (float)((double)m_used * 0.6931471805599453 + log((double)l) - p.lse_skew * (double)mx_used);
        if (p.n_splits == 1) {
          uint4* dst = reinterpret_cast<uint4*>(p.o + ((size_t)tok * p.hq + h) * D);
#pragma unroll
          for (int c = 0; c < D / 32; ++c)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int x = 8 * e;
              dst[c * 4 + e] = make_uint4(
                  pack_bf16x2(__uint_as_float(r[c][x]) * inv_l, __uint_as_float(r[c][x + 1]) * inv_l),
                  pack_bf16x2(__uint_as_float(r[c][x + 2]) * inv_l, __uint_as_float(r[c][x + 3]) * inv_l),
                  pack_bf16x2(__uint_as_float(r[c][x + 4]) * inv_l, __uint_as_float(r[c][x + 5]) * inv_l),
                  pack_bf16x2(__uint_as_float(r[c][x + 6]) * inv_l, __uint_as_float(r[c][x + 7]) * inv_l));
            }
          p.lse[(size_t)h * p.total_q + tok] = lse;
        } else {
          float4* dst = reinterpret_cast<float4*>(p.o_part + (((size_t)sp * p.total_q + tok) * p.hq + h) * D);
#pragma unroll
          for (int c = 0; c < D / 32; ++c)
#pragma unroll
            for (int e = 0; e < 8; ++e)
              dst[c * 8 + e] = make_float4(__uint_as_float(r[c][4 * e]) * inv_l, __uint_as_float(r[c][4 * e + 1]) * inv_l,
                                           __uint_as_float(r[c][4 * e + 2]) * inv_l,
                                           __uint_as_float(r[c][4 * e + 3]) * inv_l);
          p.lse_part[((size_t)sp * p.hq + h) * p.total_q + tok] = lse;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Combine the splits of one (token, head) row per warp:
//   LSE = m + ln sum_s exp(LSE_s - m),  O = sum_s exp(LSE_s - m) O_s / sum_s exp(LSE_s - m),
// with m = max_s LSE_s; splits with LSE_s = -inf (no visible key) contribute nothing, and a
// row with no visible key at all gets O = 0, LSE = -inf.
template <int D>
__global__ void __launch_bounds__(256) decode_combine(const float* __restrict__ o_part,
                                                      const float* __restrict__ lse_part, int n_splits,
                                                      int total_q, int hq, __nv_bfloat16* __restrict__ o,
                                                      float* __restrict__ lse) {
  constexpr int PER_LANE = D / 32;
  const int lane = threadIdx.x & 31;
  const int64_t rows = (int64_t)total_q * hq;
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t rw = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); rw < rows; rw += nwarps) {
    const int tok = (int)(rw / hq), h = (int)(rw % hq);
    float m = -INFINITY;
    for (int s = lane; s < n_splits; s += 32) m = fmaxf(m, lse_part[((size_t)s * hq + h) * total_q + tok]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    float acc[PER_LANE];
#pragma unroll
    for (int e = 0; e < PER_LANE; ++e) acc[e] = 0.f;
    float wsum = 0.f;
    if (m != -INFINITY) {
      for (int s = 0; s < n_splits; ++s) {
        const float ls = lse_part[((size_t)s * hq + h) * total_q + tok];
        if (ls == -INFINITY) continue;
        const float w = exp2f((ls - m) * kLog2e);
        wsum += w;
        const float* src = o_part + (((size_t)s * total_q + tok) * hq + h) * D + lane * PER_LANE;
#pragma unroll
        for (int e = 0; e < PER_LANE; ++e) acc[e] = fmaf(w, src[e], acc[e]);
      }
    }
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
    __nv_bfloat16* dst = o + ((size_t)tok * hq + h) * D + lane * PER_LANE;
    if constexpr (PER_LANE == 1) {
      dst[0] = __float2bfloat16_rn(acc[0] * inv);
    } else {
#pragma unroll
      for (int e = 0; e < PER_LANE; e += 2)
        *reinterpret_cast<uint32_t*>(dst + e) = pack_bf16x2(acc[e] * inv, acc[e + 1] * inv);
    }
    if (lane == 0) lse[(size_t)h * total_q + tok] = wsum > 0.f ? m + logf(wsum) : -INFINITY;
  }
}

int decode_sm_count() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  }
  return n;
}

template <int D>
cudaError_t launch_decode_d(const DecodeProblem& pb, const void* q, const void* k, const void* v, void* o,
                            float* lse, void* workspace, cudaStream_t stream) {
  using C = DecCfg<D>;
  const DecodeSplit sp = decode_split(pb);
  const int G = pb.hq / pb.hkv;
  alignas(64) CUtensorMap tq, tk, tv;
  if (!encode_tma_3d_box(&tq, q, D, pb.hq, pb.total_q, C::PANEL, G, pb.max_seqlen_q) ||
      !encode_tma_3d(&tk, k, D, pb.hkv, pb.total_k, C::PANEL, kKeys) ||
      !encode_tma_3d(&tv, v, D, pb.hkv, pb.total_k, C::PANEL, kKeys))
    return cudaErrorInvalidValue;
  DecParams p;
  p.cu_q = pb.cu_q;
  p.cu_k = pb.cu_k;
  p.seqlen_q = pb.seqlen_q;
  p.seqlen_k = pb.seqlen_k;
  p.max_seqlen_q = pb.max_seqlen_q;
  p.max_seqlen_k = pb.max_seqlen_k;
  p.total_q = pb.total_q;
  p.total_k = pb.total_k;
  p.hq = pb.hq;
  p.hkv = pb.hkv;
  p.G = G;
  p.tiles_per_split = sp.tiles_per_split;
  p.n_splits = sp.n_splits;
  p.scale_log2 = pb.scale * kLog2e;
  p.lse_skew = (double)p.scale_log2 * 0.6931471805599453 - (double)pb.scale;
  p.causal = pb.causal;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.o_part = static_cast<float*>(workspace);
  p.lse_part = sp.n_splits > 1 ? reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + sp.o_part_bytes)
                               : nullptr;
  cudaError_t e = cudaFuncSetAttribute(decode_bf16_sm100<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  {
    LaunchScope scope(K_DECODE_BF16, stream);
    decode_bf16_sm100<D><<<dim3(sp.n_splits, pb.hkv, pb.batch), kThreads, C::SMEM_BYTES, stream>>>(tq, tk, tv, p);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess || sp.n_splits == 1) return e;
  const int64_t rows = (int64_t)pb.total_q * pb.hq;
  const int blocks = (int)std::min<int64_t>((rows + 7) / 8, (int64_t)decode_sm_count() * 16);
  LaunchScope scope(K_DECODE_COMBINE, stream);
  decode_combine<D><<<blocks, 256, 0, stream>>>(p.o_part, p.lse_part, sp.n_splits, pb.total_q, pb.hq,
                                                static_cast<__nv_bfloat16*>(o), lse);
  return cudaGetLastError();
}

}  // namespace

DecodeSplit decode_split(const DecodeProblem& pb) {
  DecodeSplit s;
  const int n_kt = std::max(1, (pb.max_seqlen_k + kKeys - 1) / kKeys);   // key tiles of the longest sequence
  const int64_t units = (int64_t)pb.batch * pb.hkv;                        // (sequence, KV head) pairs
  const int sms = decode_sm_count();
  int n = pb.num_splits;
  // Varlen calls whose lengths are all within 10% of the longest (judged from the total)
  // are scheduled like equal lengths.
  const int64_t tiles = ((int64_t)pb.total_k + kKeys - 1) / kKeys + pb.batch;
  const bool ragged = pb.varlen && tiles * 10 < (int64_t)pb.batch * n_kt * 9;
  if (n <= 0) {
    if (ragged) {
      // Lengths differ and only their total is known here: splits of about a quarter of
      // an SM's average share of key tiles keep the longest sequences from setting the time.
      const int64_t share = (tiles * pb.hkv + sms - 1) / sms;
      const int tps = (int)std::max<int64_t>(8, (share + 3) / 4);
      n = (n_kt + tps - 1) / tps;
    } else {
      // Equal lengths: one CTA per SM at a time (shared memory), so the time goes as the
      // number of waves times (the tiles per split + a CTA's fixed cost, its pipeline fill
      // and epilogue, about 4 tile times on B200), plus the combine pass when split;
      // among equal costs take fewer splits.
      int64_t best = INT64_MAX;
      for (int c = 1; c <= std::min(n_kt, 64); ++c) {
        const int64_t waves = (units * c + sms - 1) / sms;
        const int64_t cost = waves * ((n_kt + c - 1) / c + 4) + (c > 1 ? 2 : 0);
        if (cost < best) {
          best = cost;
          n = c;
        }
      }
    }
  }
  n = std::max(1, std::min(n, n_kt));
  s.tiles_per_split = (n_kt + n - 1) / n;
  s.n_splits = (n_kt + s.tiles_per_split - 1) / s.tiles_per_split;
  s.o_part_bytes = s.n_splits > 1 ? (((size_t)s.n_splits * pb.total_q * pb.hq * pb.d * 4 + 255) & ~(size_t)255) : 0;
  s.workspace_bytes = s.n_splits > 1 ? s.o_part_bytes + (size_t)s.n_splits * pb.hq * pb.total_q * 4 : 0;
  return s;
}

cudaError_t launch_decode_bf16(const DecodeProblem& pb, const void* q, const void* k, const void* v, void* o,
                               float* lse, void* workspace, cudaStream_t stream) {
  if (pb.total_q == 0 || pb.batch == 0) return cudaSuccess;
  switch (pb.d) {
    case 32: return launch_decode_d<32>(pb, q, k, v, o, lse, workspace, stream);
    case 64: return launch_decode_d<64>(pb, q, k, v, o, lse, workspace, stream);
    case 128: return launch_decode_d<128>(pb, q, k, v, o, lse, workspace, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace attn
