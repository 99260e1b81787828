// bwd_sm100.cu -- exact attention backward for sm_100a (bf16 tensors): TMA + tcgen05.
//
// What it computes (the analytic gradient of O = softmax(scale Q K^T [+mask]) V):
//     D_i   = sum_c dO_ic O_ic
//     P_ij  = exp(scale S_ij - LSE_i),   S = Q K^T      (recomputed, never stored)
//     dS_ij = P_ij (dO_i . V_j - D_i)
//     dQ = scale dS K,   dK = scale dS^T Q,   dV = P^T dO
// The "FlashAttention 与高效注意力内核" tutorial, sections 反向 and 反向重算流程: the
// backward reloads Q/K/V tiles, recomputes S and P on chip from the saved statistics,
// combines them with dO, and drops every tile when it is done, so memory stays O(N).
//
// Three launches on the caller's stream:
//   1. bwd_preprocess   D = rowsum(dO o O) into the workspace and zero the fp32 dQ
//                       accumulator (HBM-bound).
//   2. bwd_main         persistent, one CTA per SM; a work item is a (128-key tile, kv
//                       head, sequence), claimed from a global counter in a fixed order.
//                       For its item the CTA keeps K_j in shared memory (two buffers: the
//                       next item's K_j loads while this one runs), V_j and dK_j, dV_j in
//                       TMEM, and walks the query tiles of every query head of the GQA
//                       group (so dK/dV need no atomics).  Per query tile i (BM rows):
//                         S^T  = K_j Q_i^T            (tcgen05, TMEM fp32)
//                         dP^T = V_j dO_i^T           (tcgen05, A = V_j from TMEM)
//                         P^T, dS^T on the compute warpgroup, one key row per thread,
//                           written back as bf16 over S^T / dP^T, dS^T also to SMEM
//                         dV  += P^T dO_i             (A from TMEM)
//                         dK  += dS^T Q_i             (A from TMEM)
//                         dQ_i partial                (A, B from SMEM)
//                       and a drain warpgroup reads each dQ_i partial out of TMEM, stages
//                       it in an fp32 SMEM tile and adds it into the fp32 accumulator with
//                       a bulk tensor reduction (cp.reduce.async.bulk.tensor, in L2).
//   3. bwd_dq_convert   dQ = bf16(scale * accumulator) (HBM-bound).
//
// dQ strategy.  Each (key tile, query tile) pair contributes a BM x d partial of dQ_i;
// the CTA that owns the key tile adds it into an fp32 accumulator (reductions in L2).  The
// alternative -- a second, query-major kernel -- would recompute S and dP (7 matrix
// products per tile instead of 5, 40% more tensor work); the reduction traffic instead
// goes to L2 (the accumulator of one head, N*d*4 bytes, stays L2-resident): the drain
// stages each partial in an fp32 SMEM tile and adds it with bulk tensor reductions.
//
// TMEM shapes.  d = 128 uses BM = 64 query rows per step and forms the transpose
// dQ_i^T = K_j^T dS^T (M = d = 128, N = 64), which fits S^T (64) + dP^T (64) + dV (128)
// + dK (128) + two dQ^T buffers (2 x 64) = 512 columns.  d <= 64 uses BM = 128 and
// dQ_i = dS K_j (M = 128 query rows, N = d): 128 + 128 + 4 d <= 512 columns.
//
// Warp roles (448 threads): two compute warpgroups, each owning half of the query columns
// of every step (P^T, dS^T) and one of the dK / dV epilogues; a dQ drain warpgroup (which
// also loads each item's V_j into TMEM, during the previous item's epilogue); a TMA
// producer warp that claims the items
// (+ LSE / D rows into SMEM, one step ahead); an MMA issuer warp.  Across items the
// pipelines keep running: the next item's K_j and first Q / dO tiles load during the
// current item, and its first products start while the epilogue drains dK / dV.
#include "kernels.h"
#include "sm100.cuh"

namespace attn {

namespace {

constexpr int kKeys = 128;   // keys per CTA == TMEM lanes
constexpr int kItemSlots = 4;  // ring of work-item indices the producer hands to the other roles
constexpr int kThreads = 448;
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct BwdCfg {
  static constexpr bool DQT = (D == 128);          // dQ^T form (see file comment)
  static constexpr bool VT = true;                // V_j held in TMEM, dP^T as a TS product
  static constexpr int STAGES = DQT ? 3 : 2;      // Q_i / dO_i / LSE_i / D_i ring depth
  // K_j (and V_j when it is not in TMEM) buffers: two, so the next work item's tile loads
  // while the current one runs.
  static constexpr int KV_BUFS = 2;
  static constexpr int BM = DQT ? 64 : 128;       // query rows per step
  static constexpr int HALF = BM / 2;             // query columns per compute warpgroup
  static constexpr int SW = D >= 64 ? 128 : 64;   // swizzle span of Q/K/V/dO rows (bytes)
  static constexpr int PANEL = SW / 2;
  static constexpr int NPANEL = D / PANEL;
  static constexpr uint32_t SWZ = SW == 128 ? 2u : 4u;
  static constexpr int SBO = 8 * SW;
  static constexpr int KSTEPS_PER_PANEL = SW / 32;
  static constexpr int KV_PANEL_BYTES = kKeys * SW;   // panel of a 128-row K or V tile
  static constexpr int KV_TILE_BYTES = kKeys * D * 2;
  static constexpr int Q_PANEL_BYTES = BM * SW;       // panel of a BM-row Q or dO tile
  static constexpr int Q_TILE_BYTES = BM * D * 2;
  static constexpr int DS_PANEL_BYTES = kKeys * 128;  // dS^T: 128 key rows x 64 queries (bf16)
  static constexpr int DS_BYTES = kKeys * BM * 2;
  // TMEM columns.  V_j (bf16 pairs, D/2 columns) is the A operand of dP^T; one dP^T
  // buffer.  d = 128:  V [0,64) S^T [64,128) dP^T [128,192) dV [192,320) dK [320,448)
  // dQ^T [448,512).  d = 64:  S^T [0,128) dP^T [128,256) dV [256,320) dK [320,384)
  // dQ [384,448) V [448,480).  d = 32: S^T, dP^T as for d = 64, dV [256,288) dK [288,320),
  // two dQ slots [320,384), V [384,400).
  static constexpr int NDPT = (DQT && !VT) ? 2 : 1;  // dP^T buffers
  static constexpr int NDQ = (DQT || D == 64) ? 1 : 2;   // dQ slots (d = 64: room for V)
  static constexpr int V_COLS = VT ? D / 2 : 0;      // V_j as a bf16 A operand: D/2 columns
  // d = 128 puts V first; d <= 64 after the accumulators (every accumulator 64-aligned)
  static constexpr int T_ST = DQT ? V_COLS : 0;
  static constexpr int T_DPT = T_ST + BM;            // dP^T buffer b at T_DPT + b * BM
  static constexpr int T_DV = T_DPT + NDPT * BM;
  static constexpr int T_DK = T_DV + D;
  static constexpr int T_DQ = T_DK + D;              // NDQ slots of DQ_COLS
  static constexpr int DQ_COLS = DQT ? BM : D;
  static constexpr int T_V = DQT ? 0 : T_DQ + NDQ * DQ_COLS;
  static_assert(T_DQ + NDQ * DQ_COLS + (DQT ? 0 : V_COLS) <= 512, "TMEM budget");
  // shared memory map (offsets from the 1024-aligned base)
  static constexpr int KVB_BYTES = (VT ? 1 : 2) * KV_TILE_BYTES;   // one K (+ V) buffer
  static constexpr int O_K = 0;                                 // buffer b at O_K + b * KVB_BYTES
  static constexpr int O_V = O_K + KV_TILE_BYTES;               // inside a buffer
  static constexpr int O_Q = O_K + KV_BUFS * KVB_BYTES;         // STAGES
  static constexpr int O_DO = O_Q + STAGES * Q_TILE_BYTES;      // STAGES
  static constexpr int O_DS = O_DO + STAGES * Q_TILE_BYTES;     // 2 buffers
  // LSE_i * log2 e and D_i rows live in LSLOTS slots (slot n % LSLOTS for step n), each
  // with its own full barrier that the compute warpgroups observe phase by phase.
  static constexpr int LSLOTS = 6;
  static_assert(LSLOTS >= STAGES, "an LSE slot must outlive the Q stage of its step");
  static constexpr int O_LSE = O_DS + 2 * DS_BYTES;            // LSLOTS x BM floats
  static constexpr int O_DD = O_LSE + LSLOTS * BM * 4;         // LSLOTS x BM floats
  // dQ staging tile for the bulk reduction, [BM query rows][d] fp32.  d = 128: plain
  // row-major (written column-wise, one feature per thread).  d <= 64: 32-float panels
  // with the 128-byte swizzle (written row-wise, one query row per thread).
  static constexpr int STG_ALIGN = DQT ? 128 : 1024;            // swizzled tiles need 1024
  static constexpr int O_STG = (O_DD + LSLOTS * BM * 4 + STG_ALIGN - 1) & ~(STG_ALIGN - 1);
  static constexpr int STG_PANEL_BYTES = BM * 128;              // d <= 64: [BM rows][32 floats]
  static constexpr int STG_ROWS = DQT ? 32 : BM;                // d = 128: two halves of 32 rows
  static constexpr int STG_BYTES = STG_ROWS * D * 4;
  static constexpr int O_BAR = O_STG + STG_BYTES;
  // barriers
  static constexpr int B_KFULL = 0;                  // KV_BUFS (2 reserved)
  static constexpr int B_KEMPTY = 2;                 // KV_BUFS (2 reserved)
  static constexpr int B_QFULL = 4;                  // STAGES
  static constexpr int B_QEMPTY = B_QFULL + STAGES;  // STAGES
  static constexpr int B_LFULL = B_QEMPTY + STAGES;  // LSLOTS
  static constexpr int B_ST = B_LFULL + LSLOTS;
  static constexpr int B_DPT = B_ST + 1;             // NDPT (2 slots reserved)
  static constexpr int B_PT = B_DPT + 2;
  static constexpr int B_DS = B_PT + 1;
  static constexpr int B_DSFREE = B_DS + 1;          // 2
  static constexpr int B_DQFULL = B_DSFREE + 2;      // 2
  static constexpr int B_DQEMPTY = B_DQFULL + 2;     // 2
  static constexpr int B_DONE = B_DQEMPTY + 2;
  static constexpr int B_VT = B_DONE + 1;            // V_j written into TMEM
  static constexpr int B_EPI = B_VT + 1;             // dK, dV read out of TMEM
  static constexpr int B_IFULL = B_EPI + 1;          // kItemSlots: item index written
  static constexpr int B_IEMPTY = B_IFULL + kItemSlots;   // kItemSlots: read by every role
  static constexpr int B_DRAIN = B_IEMPTY + kItemSlots;   // the MMA issuer's completion at exit
  static constexpr int NBARS = B_DRAIN + 1;
  // after the barriers: TMEM address, abort flag, the item-index ring
  static constexpr int SMEM_BYTES = 1024 + O_BAR + NBARS * 8 + 8 + 4 * kItemSlots;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  // the dK / dV epilogue stages 32 rows per compute warp in the finished item's K buffer:
  // row segments of up to 128 bytes, as much as the buffer holds
  static constexpr int EPI_ROWB_CAP = KVB_BYTES / (8 * 32);
  static constexpr int EPI_ROWB = (D * 2 < 128 ? D * 2 : 128) < EPI_ROWB_CAP ? (D * 2 < 128 ? D * 2 : 128)
                                                                             : EPI_ROWB_CAP;
  static_assert(EPI_ROWB >= 32 && 8 * 32 * EPI_ROWB <= KVB_BYTES, "epilogue staging fits in a K buffer");
};

struct BwdParams {
  const int32_t* cu_seqlens;
  int32_t seqlen, max_seqlen, total_tokens, hq, hkv;
  float scale;
  float scale_log2;
  int32_t causal;
  const float* lse;      // [hq, T]
  const float* dd;       // [hq, T]
  const __nv_bfloat16* v;   // [T, hkv, d] (read directly when V_j lives in TMEM)
  int32_t batch, n_kt, n_items;   // work items: (key tile, kv head, sequence)
  int32_t heads_per_group;         // causal order: heads whose Q / dO stream fits in L2
  int* item_counter;               // next unclaimed item (zeroed by the preprocess kernel)
  float* dq_acc;         // [T, hq, d]
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  // accumulate mode: dK and dV are added into these float32 [T, hkv, d] tensors (and dQ,
  // scaled, into dq_acc, which is then the caller's) instead of being written as bf16
  int32_t accumulate;
  float dq_mul;          // factor on each dQ partial: scale in accumulate mode, else 1
  float* dk_acc;
  float* dv_acc;
};

// Enumerates the (query head, query tile) steps of one CTA in a fixed order.
struct StepIter {
  int G, i_begin, n_q, steps_per_head;
  __device__ void head_tile(int n, int g, int* h, int* i) const {
    *h = g * G + n / steps_per_head;
    *i = i_begin + n % steps_per_head;
  }
};

// One work item: a 128-key tile of one kv head of one sequence.
struct BItem {
  int g, seq_start, len, kv0, n_steps;   // n_steps == 0: nothing to do
  StepIter it;
};

// Work item number idx.  The CTAs are persistent (one per SM) and claim items in this
// order from a global counter, so each takes the next one as soon as it is free.  With
// heads_per_group > 0 (causal, d = 128) the order is heaviest-first (key tile 0 is seen
// by every query) within groups of heads whose Q / dO stream fits in about 32 MB of L2,
// so that the items in flight share what they read and lighter items fill in at the end;
// otherwise the key tiles of one head are consecutive.
template <int BM>
__device__ __forceinline__ BItem bitem_from(const BwdParams& p, int idx) {
  BItem w;
  w.n_steps = 0;
  w.g = w.seq_start = w.len = w.kv0 = 0;
  w.it.G = w.it.i_begin = w.it.n_q = w.it.steps_per_head = 0;
  if (idx < 0 || idx >= p.n_items) return w;
  int jt, r;
  if (p.causal && p.heads_per_group > 0) {
    const int pairs = p.hkv * p.batch;
    const int per_grp = p.n_kt * p.heads_per_group;
    const int grp = idx / per_grp, rem = idx % per_grp;
    const int ng = min(p.heads_per_group, pairs - grp * p.heads_per_group);
    jt = rem / ng;
    r = grp * p.heads_per_group + rem % ng;
  } else {
    jt = idx % p.n_kt;
    r = idx / p.n_kt;
  }
  w.g = r % p.hkv;
  const int b = r / p.hkv;
  w.seq_start = p.cu_seqlens ? p.cu_seqlens[b] : b * p.seqlen;
  w.len = p.cu_seqlens ? p.cu_seqlens[b + 1] - w.seq_start : p.seqlen;
  w.kv0 = jt * kKeys;
  if (w.kv0 >= w.len) return w;
  w.it.G = p.hq / p.hkv;
  w.it.n_q = (w.len + BM - 1) / BM;
  w.it.i_begin = p.causal ? w.kv0 / BM : 0;
  w.it.steps_per_head = w.it.n_q - w.it.i_begin;
  w.n_steps = w.it.G * w.it.steps_per_head;
  return w;
}

// Byte offset of the 16-byte chunk `chunk` of row `row` inside a 128-byte-swizzled panel.
__device__ __forceinline__ uint32_t sw128_offset(int row, int chunk) {
  return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4));
}

// Warp roles (448 threads):
//   warps 0-3   compute, query columns [0, BM/2) of every step, then the dV epilogue
//   warps 4-7   compute, query columns [BM/2, BM), then the dK epilogue
//   warps 8-11  dQ drain; also loads each item's V_j into TMEM
//   warp  12    producer (TMA for K, V, Q_i, dO_i; LSE_i, D_i rows into SMEM)
//   warp  13    MMA issuer
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_bf16_sm100(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                   const __grid_constant__ CUtensorMap tmDQ, const BwdParams p) {
  using C = BwdCfg<D>;
  constexpr int BM = C::BM;
  constexpr int HALF = C::HALF;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  float* s_lse = reinterpret_cast<float*>(smem + C::O_LSE);
  float* s_dd = reinterpret_cast<float*>(smem + C::O_DD);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::O_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NBARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* s_items = reinterpret_cast<volatile int*>(tmem_slot + 2);
  auto bar = [&](int i) { return smem_u32(bars + i); };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // The producer claims items and hands their indices to the other roles through the
  // s_items ring; every role walks the same items in the same order.  Per-step barriers
  // count steps over all the CTA's items; per-item ones (K buffers, V in TMEM, done,
  // epilogue) count non-empty items.  next_item(k) returns the k-th claimed index (or
  // -1 after a failed wait); an index >= n_items ends the walk.
  auto next_item = [&](int k) -> int {
    const int slot = k % kItemSlots;
    if (!mbar_wait(bar(C::B_IFULL + slot), (k / kItemSlots) & 1, abort_flag)) return -1;
    const int idx = s_items[slot];
    __syncwarp(__activemask());
    if ((threadIdx.x & 31) == __ffs(__activemask()) - 1) mbar_arrive(bar(C::B_IEMPTY + slot));
    return idx;
  };

  if (threadIdx.x == 0) {
    // Key tiles past max_seqlen are not in the item list, so a longer sequence would lose
    // part of its gradients: report it (the items still run, on the tiles they cover).
    if (blockIdx.x == 0)
      for (int b = 0; b < p.batch; ++b) {
        const int len = p.cu_seqlens ? p.cu_seqlens[b + 1] - p.cu_seqlens[b] : p.seqlen;
        if (len > p.max_seqlen) report_error(ATTN_DEVERR_SEQLEN);
      }
    for (int i = 0; i < C::NBARS; ++i) {
      uint32_t cnt = 1;
      // warp-level arrivals: one per compute warp (PT, DS, K buffer free, epilogue read
      // out) or drain warp (DQEMPTY, V in TMEM)
      if (i == C::B_PT || i == C::B_DS || i == C::B_EPI || i == C::B_KEMPTY || i == C::B_KEMPTY + 1) cnt = 8;
      if (i == C::B_DQEMPTY || i == C::B_DQEMPTY + 1 || i == C::B_VT) cnt = 4;
      // item slots are read by the MMA warp, the 8 compute warps and the 4 drain warps
      if (i >= C::B_IEMPTY && i < C::B_IEMPTY + kItemSlots) cnt = 13;
      mbar_init(bar(i), cnt);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  if (warp == 12 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmDO);
    tma_prefetch_desc(&tmDQ);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 12) {
    // ---------------- producer: K_j (V_j) per item; Q_i, dO_i, LSE_i, D_i per step ---------
    // LSE_i * log2(e) and D_i of the next step are loaded into registers one step ahead,
    // so their global-memory latency overlaps the wait for a free stage.  Query rows past
    // the sequence get LSE = +inf (P = 0 there without a mask) and D = 0.
    constexpr int PER_LANE = BM / 32;
    float nl[PER_LANE], nd[PER_LANE];
    int ng = 0;          // steps so far (all items)
    int in = 0;          // non-empty items so far
    uint32_t kc = 0, qc = 0;   // K-buffer and Q / dO stage loads issued
    bool ok = true;
    for (int k = 0; ok; ++k) {
      // claim the next item and hand its index to the other roles
      const int slot = k % kItemSlots;
      if (!mbar_wait(bar(C::B_IEMPTY + slot), ((k / kItemSlots) & 1) ^ 1, abort_flag)) break;
      int idx = 0;
      if (lane == 0) {
        idx = atomicAdd(p.item_counter, 1);
        s_items[slot] = idx;
      }
      idx = __shfl_sync(0xffffffffu, idx, 0);
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::B_IFULL + slot));
      if (idx >= p.n_items) break;
      const BItem w = bitem_from<BM>(p, idx);
      if (w.n_steps == 0) continue;
      const int kb = in % C::KV_BUFS;
      // The buffer is free once the item that used it last has finished its epilogue.
      if (!mbar_wait(bar(C::B_KEMPTY + kb), ((in / C::KV_BUFS) & 1) ^ 1, abort_flag)) break;
      if (lane == 0) {
        const uint32_t kbase = sbase + C::O_K + kb * C::KVB_BYTES;
        mbar_arrive_expect_tx(bar(C::B_KFULL + kb), C::KVB_BYTES);
        for (int pn = 0; pn < C::NPANEL; ++pn) {
          tma_load_3d(kbase + pn * C::KV_PANEL_BYTES, &tmK, bar(C::B_KFULL + kb), pn * C::PANEL, w.g,
                      w.seq_start + w.kv0);
          if (!C::VT)
            tma_load_3d(kbase + (C::O_V - C::O_K) + pn * C::KV_PANEL_BYTES, &tmV, bar(C::B_KFULL + kb),
                        pn * C::PANEL, w.g, w.seq_start + w.kv0);
        }
      }
      ++kc;
      auto fetch = [&](int n) {
        int h, i;
        w.it.head_tile(n, w.g, &h, &i);
#pragma unroll
        for (int e = 0; e < PER_LANE; ++e) {
          const int qi = i * BM + e * 32 + lane;
          const bool in_seq = qi < w.len;
          const size_t idx = (size_t)h * p.total_tokens + w.seq_start + (in_seq ? qi : 0);
          nl[e] = in_seq ? p.lse[idx] * kLog2e : INFINITY;
          nd[e] = in_seq ? p.dd[idx] : 0.f;
        }
      };
      fetch(0);
      for (int n = 0; n < w.n_steps; ++n, ++ng) {
        const int s = ng % C::STAGES;
        const int ls = ng % C::LSLOTS;
        // Stage s is free once dK(ng - STAGES) is done; LSE slot ls was last read by step
        // ng - LSLOTS, whose dS finished before dK(ng - LSLOTS), so it is free too.
        if (!mbar_wait(bar(C::B_QEMPTY + s), ((ng / C::STAGES) & 1) ^ 1, abort_flag)) { ok = false; break; }
        int h, i;
        w.it.head_tile(n, w.g, &h, &i);
        const int q0 = i * BM;
#pragma unroll
        for (int e = 0; e < PER_LANE; ++e) {
          s_lse[ls * BM + e * 32 + lane] = nl[e];
          s_dd[ls * BM + e * 32 + lane] = nd[e];
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(C::B_LFULL + ls));
        if (n + 1 < w.n_steps) fetch(n + 1);
        if (lane == 0) {
          mbar_arrive_expect_tx(bar(C::B_QFULL + s), 2 * C::Q_TILE_BYTES);
          for (int pn = 0; pn < C::NPANEL; ++pn) {
            tma_load_3d(sbase + C::O_Q + s * C::Q_TILE_BYTES + pn * C::Q_PANEL_BYTES, &tmQ, bar(C::B_QFULL + s),
                        pn * C::PANEL, h, w.seq_start + q0);
            tma_load_3d(sbase + C::O_DO + s * C::Q_TILE_BYTES + pn * C::Q_PANEL_BYTES, &tmDO, bar(C::B_QFULL + s),
                        pn * C::PANEL, h, w.seq_start + q0);
          }
        }
        ++qc;
      }
      ++in;
    }
    // Every load issued here lands before the CTA releases its memory, also when another
    // role gave up waiting: only the last load of each buffer / stage can still be in flight.
    if (lane == 0) {
      for (uint32_t i = kc > (uint32_t)C::KV_BUFS ? kc - C::KV_BUFS : 0; i < kc; ++i)
        mbar_wait_drain(bar(C::B_KFULL + i % C::KV_BUFS), (i / C::KV_BUFS) & 1);
      for (uint32_t i = qc > (uint32_t)C::STAGES ? qc - C::STAGES : 0; i < qc; ++i)
        mbar_wait_drain(bar(C::B_QFULL + i % C::STAGES), (i / C::STAGES) & 1);
    }
  } else if (warp == 13) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t id_sdp = idesc_bf16_f32(kKeys, BM, false, false);   // K Q^T, V dO^T
      const uint32_t id_grad = idesc_bf16_f32(kKeys, D, false, true);    // P^T dO, dS^T Q
      const uint32_t id_dq = C::DQT ? idesc_bf16_f32(D, BM, true, true)  // K^T dS^T
                                    : idesc_bf16_f32(BM, D, true, true); // dS K
      auto kmajor_off = [&](int kk, int panel_bytes) {
        return (uint32_t)((kk / C::KSTEPS_PER_PANEL) * panel_bytes + (kk % C::KSTEPS_PER_PANEL) * 32);
      };
      // Every operand descriptor is a base descriptor (computed once, or once per ring
      // stage) advanced by a compile-time offset, so issuing one MMA takes a few
      // instructions; the issue rate of this single thread bounds the tensor core here.
      // K / V descriptors of buffer 0; buffer kb adds kb * KVB_BYTES
      const uint64_t k_kmaj0 = smem_desc(sbase + C::O_K, 16, C::SBO, C::SWZ);               // K, K-major
      const uint64_t v_kmaj0 = smem_desc(sbase + C::O_V, 16, C::SBO, C::SWZ);               // V, K-major
      const uint64_t k_mn0 = smem_desc(sbase + C::O_K, C::KV_PANEL_BYTES, C::SBO, C::SWZ);  // K^T operand
      uint64_t k_kmaj = k_kmaj0, v_kmaj = v_kmaj0, k_mn = k_mn0;
      const uint64_t q_kmaj = smem_desc(sbase + C::O_Q, 16, C::SBO, C::SWZ);
      const uint64_t do_kmaj = smem_desc(sbase + C::O_DO, 16, C::SBO, C::SWZ);
      const uint64_t q_mn = smem_desc(sbase + C::O_Q, C::Q_PANEL_BYTES, C::SBO, C::SWZ);
      const uint64_t do_mn = smem_desc(sbase + C::O_DO, C::Q_PANEL_BYTES, C::SBO, C::SWZ);
      const uint64_t ds_desc = smem_desc(sbase + C::O_DS, C::DS_PANEL_BYTES, 1024, 2u);
      auto stage = [&](uint64_t base, int s) { return desc_advance(base, (uint32_t)s * C::Q_TILE_BYTES); };
      // X_tile (128 keys) times Y_i^T (BM rows), both K-major over d
      auto issue_sdp = [&](uint64_t x, uint64_t y, uint32_t d_col) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tmem + d_col, desc_advance(x, kmajor_off(kk, C::KV_PANEL_BYTES)),
                 desc_advance(y, kmajor_off(kk, C::Q_PANEL_BYTES)), id_sdp, kk > 0 ? 1u : 0u);
      };
      // D[128 keys x d] += A^T(TMEM, bf16 over BM queries) * Y_i (BM x d, MN-major).
      // Each compute warpgroup packs its half of the queries into the first columns of
      // its own half of the fp32 region, so queries [h*HALF, (h+1)*HALF) sit at columns
      // h*HALF + (q - h*HALF)/2.
      auto issue_grad = [&](uint32_t a_col, uint64_t y, uint32_t d_col, bool acc) {
#pragma unroll
        for (int kk = 0; kk < BM / 16; ++kk) {
          const int qb = kk * 16;
          const int hh = qb / HALF;
          const uint32_t col = a_col + hh * HALF + (qb - hh * HALF) / 2;
          mma_ts(tmem + d_col, tmem + col, desc_advance(y, kk * 16 * C::SW), id_grad, (acc || kk > 0) ? 1u : 0u);
        }
      };
      // dP^T = V_j dO_i^T: from shared memory, or with V_j (A) read out of TMEM
      auto issue_dpt = [&](uint64_t y, uint32_t d_col) {
        if (C::VT) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_ts(tmem + d_col, tmem + C::T_V + kk * 8, desc_advance(y, kmajor_off(kk, C::Q_PANEL_BYTES)), id_sdp,
                   kk > 0 ? 1u : 0u);
        } else {
          issue_sdp(v_kmaj, y, d_col);
        }
      };
      auto issue_dq = [&](int dsbuf, uint32_t d_col) {
        const uint64_t ds = desc_advance(ds_desc, (uint32_t)dsbuf * C::DS_BYTES);
#pragma unroll
        for (int kk = 0; kk < kKeys / 16; ++kk) {
          const uint64_t kd = desc_advance(k_mn, kk * 16 * C::SW);
          const uint64_t sd = desc_advance(ds, kk * 16 * 128);
          if (C::DQT)
            mma_ss(tmem + d_col, kd, sd, id_dq, kk > 0 ? 1u : 0u);
          else
            mma_ss(tmem + d_col, sd, kd, id_dq, kk > 0 ? 1u : 0u);
        }
      };
      int ng0 = 0;         // steps before the current item (all items)
      int in = 0;          // non-empty items so far
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int idx = next_item(k);
        if (idx < 0 || idx >= p.n_items) break;
        const BItem w = bitem_from<BM>(p, idx);
        if (w.n_steps == 0) continue;
        const int kb = in % C::KV_BUFS;
        k_kmaj = desc_advance(k_kmaj0, (uint32_t)kb * C::KVB_BYTES);
        v_kmaj = desc_advance(v_kmaj0, (uint32_t)kb * C::KVB_BYTES);
        k_mn = desc_advance(k_mn0, (uint32_t)kb * C::KVB_BYTES);
        const int s0 = ng0 % C::STAGES;
        ok = mbar_wait(bar(C::B_KFULL + kb), (in / C::KV_BUFS) & 1, abort_flag) &&
             mbar_wait(bar(C::B_QFULL + s0), (ng0 / C::STAGES) & 1, abort_flag);
        if (ok) {
          tc_fence_after();
          issue_sdp(k_kmaj, stage(q_kmaj, s0), C::T_ST);
          mma_commit(bar(C::B_ST));
          // V_j of this item in TMEM (the drain loads it once the previous item's dP^T are done)
          ok = !C::VT || mbar_wait(bar(C::B_VT), in & 1, abort_flag);
        }
        if (ok) {
          tc_fence_after();
          issue_dpt(stage(do_kmaj, s0), C::T_DPT + (C::NDPT == 2 ? (ng0 & 1) * BM : 0));
          mma_commit(bar(C::B_DPT + (C::NDPT == 2 ? (ng0 & 1) : 0)));
        }
        // Order per step n (global step ng; dP^T buffer db = ng & 1 when NDPT == 2, else 0):
        //   [PT(ng)] dV(ng); S^T(ng+1); NDPT == 2: dP^T(ng+1) into the other buffer;
        //   [DS(ng)] dK(ng) (reads dS^T(ng) from buffer db); [dQ slot free] dQ(ng);
        //   NDPT == 1: dP^T(ng+1) here, once dK(ng) has been issued.
        // The first dV / dK of an item overwrite the accumulators, so they wait until the
        // previous item's epilogue has read them out.
        // Every barrier this thread depends on inside a step is checked with mbar_test one
        // MMA group before the group that needs it (mbar_wait only if it had not completed
        // then): the tensor pipe's queue is short, and a check that waits for its own
        // shared-memory round trip leaves it idle.
        bool pt_ready = false;   // P^T(ng) seen complete by the check started in the last step
        for (int n = 0; ok && n < w.n_steps; ++n) {
          const int ng = ng0 + n;
          const int s = ng % C::STAGES;
          const int s1 = (ng + 1) % C::STAGES;
          const int b2 = ng & 1;
          const int db = C::NDPT == 2 ? b2 : 0;
          const int db1 = C::NDPT == 2 ? (b2 ^ 1) : 0;
          const int qslot = C::NDQ == 2 ? b2 : 0;
          const uint32_t qpar = C::NDQ == 2 ? (((ng >> 1) & 1) ^ 1) : (uint32_t)((ng & 1) ^ 1);
          const bool more = n + 1 < w.n_steps;
          if (!pt_ready && !mbar_wait(bar(C::B_PT), ng & 1, abort_flag)) { ok = false; break; }
          if (n == 0 && in > 0 && !mbar_wait(bar(C::B_EPI), (in - 1) & 1, abort_flag)) { ok = false; break; }
          const bool q_ready = !more || mbar_test(bar(C::B_QFULL + s1), ((ng + 1) / C::STAGES) & 1);
          tc_fence_after();
          issue_grad(C::T_ST, stage(do_mn, s), C::T_DV, n > 0);                 // dV += P^T dO
          const bool ds_ready = mbar_test(bar(C::B_DS), ng & 1);
          if (more) {
            if (!q_ready && !mbar_wait(bar(C::B_QFULL + s1), ((ng + 1) / C::STAGES) & 1, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_sdp(k_kmaj, stage(q_kmaj, s1), C::T_ST);                      // S^T for the next step
            mma_commit(bar(C::B_ST));
            if (C::NDPT == 2) {
              issue_dpt(stage(do_kmaj, s1), C::T_DPT + db1 * BM);               // dP^T(ng+1)
              mma_commit(bar(C::B_DPT + db1));
            }
          }
          if (!ds_ready && !mbar_wait(bar(C::B_DS), ng & 1, abort_flag)) { ok = false; break; }
          const bool dq_ready = mbar_test(bar(C::B_DQEMPTY + qslot), qpar);
          tc_fence_after();
          issue_grad(C::T_DPT + db * BM, stage(q_mn, s), C::T_DK, n > 0);       // dK += dS^T Q
          mma_commit(bar(C::B_QEMPTY + s));
          if (!dq_ready && !mbar_wait(bar(C::B_DQEMPTY + qslot), qpar, abort_flag)) { ok = false; break; }
          tc_fence_after();
          issue_dq(b2, C::T_DQ + qslot * C::DQ_COLS);                           // dQ_i partial
          mma_commit(bar(C::B_DQFULL + qslot));
          mma_commit(bar(C::B_DSFREE + b2));
          pt_ready = more && mbar_test(bar(C::B_PT), (ng + 1) & 1);
          if (C::NDPT == 1 && more) {
            issue_dpt(stage(do_kmaj, s1), C::T_DPT);                            // dP^T for the next step
            mma_commit(bar(C::B_DPT));
          }
        }
        mma_commit(bar(C::B_DONE));    // every product of this item (dK, dV final)
        ng0 += w.n_steps;
        ++in;
      }
      // every MMA issued here has completed before the CTA frees Tensor Memory
      mma_commit(bar(C::B_DRAIN));
      mbar_wait_drain(bar(C::B_DRAIN), 0);
    }
  } else if (warp < 8) {
    // ---------------- compute: P^T, dS^T for one key row and half of the query columns ----
    const int half = warp >> 2;                   // 0: columns [0, HALF), 1: [HALF, BM)
    const int lane_base = (warp & 3) * 32;
    const int kr = lane_base + lane;              // key row inside the tile
    const int c0 = half * HALF;                   // first query column of this thread
    const uint32_t trow = tmem + ((uint32_t)lane_base << 16);
    const float sl2 = p.scale_log2;
    int ng0 = 0;         // steps before the current item (all items)
    int in = 0;          // non-empty items so far
    bool ok = true;
    for (int k = 0; ok; ++k) {
    const int idx = next_item(k);
    if (idx < 0 || idx >= p.n_items) break;
    const BItem w = bitem_from<BM>(p, idx);
    if (w.n_steps == 0) continue;
    const int g = w.g, seq_start = w.seq_start, len = w.len, kv0 = w.kv0;
    const int kj = kv0 + kr;                      // key index inside the sequence
    for (int n = 0; n < w.n_steps; ++n) {
      const int ng = ng0 + n;
      const int ls = ng % C::LSLOTS;
      const int b2 = ng & 1;
      const int db = C::NDPT == 2 ? b2 : 0;                           // dP^T buffer
      const uint32_t dpar = C::NDPT == 2 ? ((ng >> 1) & 1) : (uint32_t)(ng & 1);
      const uint32_t t_dpt = C::T_DPT + db * BM;
      int h, i;
      w.it.head_tile(n, g, &h, &i);
      const int q0 = i * BM;
      // Columns c < c_lo are hidden by the causal mask; a key past the sequence hides all.
      // (Query rows past the sequence carry LSE = +inf, so they come out as P = 0.)
      int c_lo = p.causal ? kj - q0 : 0;
      if (kj >= len) c_lo = BM;
      const bool masked = c_lo > c0;
      if (!mbar_wait(bar(C::B_LFULL + ls), (ng / C::LSLOTS) & 1, abort_flag)) { ok = false; break; }
      if (!mbar_wait(bar(C::B_ST), ng & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      const float4* lse4 = reinterpret_cast<const float4*>(s_lse + ls * BM + c0);
      const float4* dd4 = reinterpret_cast<const float4*>(s_dd + ls * BM + c0);
      float pr[HALF];
#pragma unroll
      for (int cb = 0; cb < HALF; cb += 32) {
        uint32_t r[32];
        tmem_ld32(trow + C::T_ST + c0 + cb, r);
        tmem_wait_ld();
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
          const float4 l4 = lse4[(cb >> 2) + e4];
          const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int e = e4 * 4 + u;
            pr[cb + e] = ex2(fmaf(__uint_as_float(r[e]), sl2, -lv[u]));
          }
        }
      }
      if (masked) {
#pragma unroll
        for (int c = 0; c < HALF; ++c)
          if (c0 + c < c_lo) pr[c] = 0.f;
      }
#pragma unroll
      for (int cb = 0; cb < HALF; cb += 32) {
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) w[e] = pack_bf16x2(pr[cb + 2 * e], pr[cb + 2 * e + 1]);
        tmem_st16(trow + C::T_ST + c0 + cb / 2, w);   // inside this warpgroup's own columns
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::B_PT));
      // dS^T = P^T o (dP^T - D): to TMEM (over dP^T) and to the swizzled SMEM buffer
      if (!mbar_wait(bar(C::B_DSFREE + b2), ((ng >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
      if (!mbar_wait(bar(C::B_DPT + db), dpar, abort_flag)) { ok = false; break; }
      tc_fence_after();
      uint8_t* ds_smem = smem + C::O_DS + b2 * C::DS_BYTES;
#pragma unroll
      for (int cb = 0; cb < HALF; cb += 32) {
        uint32_t r[32];
        tmem_ld32(trow + t_dpt + c0 + cb, r);
        tmem_wait_ld();
        uint32_t w[16];
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
          const float4 d4 = dd4[(cb >> 2) + e4];
          const int e = e4 * 4;
          w[2 * e4] = pack_bf16x2(pr[cb + e] * (__uint_as_float(r[e]) - d4.x),
                                  pr[cb + e + 1] * (__uint_as_float(r[e + 1]) - d4.y));
          w[2 * e4 + 1] = pack_bf16x2(pr[cb + e + 2] * (__uint_as_float(r[e + 2]) - d4.z),
                                      pr[cb + e + 3] * (__uint_as_float(r[e + 3]) - d4.w));
        }
        tmem_st16(trow + t_dpt + c0 + cb / 2, w);
        // queries c0+cb .. +31 live in panel (c0+cb)/64, 16-byte chunks ((c0+cb)%64)/8 .. +3
        uint8_t* panel = ds_smem + ((c0 + cb) / 64) * C::DS_PANEL_BYTES;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          const int chunk = ((c0 + cb) % 64) / 8 + ch;
          *reinterpret_cast<uint4*>(panel + sw128_offset(kr, chunk)) =
              make_uint4(w[4 * ch], w[4 * ch + 1], w[4 * ch + 2], w[4 * ch + 3]);
        }
      }
      fence_proxy_async_smem();
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::B_DS));
    }
    // ---------------- epilogue: warps 0-3 write dV, warps 4-7 write dK = scale * acc ------
    if (!ok || !mbar_wait(bar(C::B_DONE), in & 1, abort_flag)) { ok = false; break; }
    if (p.accumulate) {
      tc_fence_after();
      // float32 read-add-write of this thread's key row (each key row of the call belongs to
      // exactly one item, so no other CTA touches it)
      float* acc = half == 0 ? p.dv_acc : p.dk_acc;
      const float mul = half == 0 ? 1.f : p.scale;
      const uint32_t col = half == 0 ? C::T_DV : C::T_DK;
      const bool in_seq = kj < len;
      float4* row = reinterpret_cast<float4*>(acc + ((size_t)(seq_start + (in_seq ? kj : 0)) * p.hkv + g) * D);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(trow + col + c * 32, r);
        tmem_wait_ld();
        if (in_seq) {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            float4 a = row[c * 8 + e];
            a.x += __uint_as_float(r[4 * e]) * mul;
            a.y += __uint_as_float(r[4 * e + 1]) * mul;
            a.z += __uint_as_float(r[4 * e + 2]) * mul;
            a.w += __uint_as_float(r[4 * e + 3]) * mul;
            row[c * 8 + e] = a;
          }
        }
      }
      const int kb = in % C::KV_BUFS;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(bar(C::B_EPI));
        mbar_arrive(bar(C::B_KEMPTY + kb));
      }
    } else {
      tc_fence_after();
      // Every product of the item has completed, so its K buffer is idle: each warp stages
      // its 32 rows there (half a row per pass at d = 128) and stores whole 128-byte row
      // segments per instruction instead of 32 scattered 16-byte pieces.  Chunk ch of
      // staged row r sits at ch ^ (r % CH): conflict-free row writes and segment reads.
      constexpr int ROWB = C::EPI_ROWB;
      constexpr int COLS = ROWB / 2;               // bf16 columns per pass
      constexpr int CH = ROWB / 16;                // 16-byte chunks per staged row
      constexpr int RPI = 32 / CH;                 // rows per coalesced store instruction
      const int kb = in % C::KV_BUFS;
      uint8_t* stg = smem + C::O_K + kb * C::KVB_BYTES + warp * 32 * ROWB;
      __nv_bfloat16* base = half == 0 ? p.dv : p.dk;
      const float mul = half == 0 ? 1.f : p.scale;
      const uint32_t col = half == 0 ? C::T_DV : C::T_DK;
      const int key0 = kv0 + lane_base;            // key index of the warp's first row
#pragma unroll
      for (int pass = 0; pass < D * 2 / ROWB; ++pass) {
        uint32_t w[COLS / 2];
        if constexpr (COLS >= 32) {
#pragma unroll
          for (int c = 0; c < COLS / 32; ++c) {
            uint32_t r[32];
            tmem_ld32(trow + col + pass * COLS + c * 32, r);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e)
              w[c * 16 + e] = pack_bf16x2(__uint_as_float(r[2 * e]) * mul, __uint_as_float(r[2 * e + 1]) * mul);
          }
        } else {   // 16 columns per pass
          uint32_t r[16];
          tmem_ld16(trow + col + pass * COLS, r);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 8; ++e)
            w[e] = pack_bf16x2(__uint_as_float(r[2 * e]) * mul, __uint_as_float(r[2 * e + 1]) * mul);
        }
#pragma unroll
        for (int ch = 0; ch < CH; ++ch)
          *reinterpret_cast<uint4*>(stg + lane * ROWB + ((ch ^ (lane % CH)) << 4)) =
              make_uint4(w[4 * ch], w[4 * ch + 1], w[4 * ch + 2], w[4 * ch + 3]);
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 32 / RPI; ++i) {
          const int r = i * RPI + lane / CH;
          const int ch = lane % CH;
          const uint4 v = *reinterpret_cast<const uint4*>(stg + r * ROWB + ((ch ^ (r % CH)) << 4));
          if (key0 + r < len)
            *reinterpret_cast<uint4*>(base + ((size_t)(seq_start + key0 + r) * p.hkv + g) * D + pass * COLS + ch * 8) = v;
        }
        __syncwarp();
      }
      // dK / dV have been read out of TMEM: the next item's first products may overwrite
      // them.  The K buffer is free for the producer once these generic accesses are
      // ordered before its next (async-proxy) write.
      tc_fence_before();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(bar(C::B_EPI));
        mbar_arrive(bar(C::B_KEMPTY + kb));
      }
    }
    ng0 += w.n_steps;
    ++in;
    }
  } else if (warp < 12) {
    // ---------------- dQ drain: TMEM partial -> staging tile -> bulk reduction into the accumulator
    const int lane_base = (warp & 3) * 32;
    const uint32_t trow = tmem + ((uint32_t)lane_base << 16);
    int ng = 0;          // steps so far (all items)
    bool ok = true;
    for (int k = 0; ok; ++k) {
    const int idx = next_item(k);
    if (idx < 0 || idx >= p.n_items) break;
    const BItem w = bitem_from<BM>(p, idx);
    const int seq_start = w.seq_start;
    if (C::VT && w.n_steps > 0) {
      // V_j into TMEM, row kr = this thread's lane: bf16 pairs as they lie in memory
      // (element 2c in the low half of column c) form the A operand of dP^T; rows past the
      // sequence are zero.  The drain does it (not the compute warps, which are writing the
      // previous item's dK / dV out by now): V's columns are free once it has read the
      // previous item's last dQ partial, whose completion follows every dP^T of that item.
      const int kj = w.kv0 + lane_base + lane;
      const uint4* vrow = reinterpret_cast<const uint4*>(p.v + ((size_t)(seq_start + kj) * p.hkv + w.g) * D);
      if constexpr (C::V_COLS >= 32) {
#pragma unroll
        for (int cb = 0; cb < C::V_COLS; cb += 32) {
          uint32_t vw[32];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const uint4 x = kj < w.len ? vrow[cb / 4 + e] : make_uint4(0u, 0u, 0u, 0u);
            vw[4 * e] = x.x;
            vw[4 * e + 1] = x.y;
            vw[4 * e + 2] = x.z;
            vw[4 * e + 3] = x.w;
          }
          tmem_st32(trow + C::T_V + cb, vw);
        }
      } else {   // d = 32: a 64-byte row, 16 columns
        uint32_t vw[16];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint4 x = kj < w.len ? vrow[e] : make_uint4(0u, 0u, 0u, 0u);
          vw[4 * e] = x.x;
          vw[4 * e + 1] = x.y;
          vw[4 * e + 2] = x.z;
          vw[4 * e + 3] = x.w;
        }
        tmem_st16(trow + C::T_V, vw);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::B_VT));
    }
    for (int n = 0; n < w.n_steps; ++n, ++ng) {
      const int b2 = C::NDQ == 2 ? (ng & 1) : 0;                   // dQ slot
      const uint32_t par = C::NDQ == 2 ? ((ng >> 1) & 1) : (uint32_t)(ng & 1);
      int h, i;
      w.it.head_tile(n, w.g, &h, &i);
      const int q0 = i * BM;
      if (!mbar_wait(bar(C::B_DQFULL + b2), par, abort_flag)) { ok = false; break; }
      tc_fence_after();
      uint32_t r[C::DQ_COLS / 32][32];
#pragma unroll
      for (int cb = 0; cb < C::DQ_COLS / 32; ++cb) tmem_ld32(trow + C::T_DQ + b2 * C::DQ_COLS + cb * 32, r[cb]);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::B_DQEMPTY + b2));
      if (C::DQT) {
        // lane = feature c, registers = the BM query rows of this step.  The partial is
        // transposed into a [BM][d] fp32 staging tile and added into the accumulator by
        // one bulk tensor reduction (query rows past the sequence carry exact zeros).
        // (Per-lane red.global.add from registers would skip shared memory but measured
        // well below the bulk reduction's throughput.)
        const int c = lane_base + lane;
        float* stg = reinterpret_cast<float*>(smem + C::O_STG);
#pragma unroll
        for (int part = 0; part < BM / C::STG_ROWS; ++part) {
          if (warp == 8 && lane == 0) bulk_wait_group_read0();   // previous reduce has read the tile
          named_barrier_sync(1, 128);
#pragma unroll
          for (int e = 0; e < C::STG_ROWS; ++e) {
            const int row = part * C::STG_ROWS + e;
            stg[e * D + c] = __uint_as_float(r[row / 32][row % 32]) * p.dq_mul;
          }
          fence_proxy_async_smem();
          named_barrier_sync(1, 128);
          if (warp == 8 && lane == 0) {
            tma_reduce_add_3d(&tmDQ, sbase + C::O_STG, 0, h, seq_start + q0 + part * C::STG_ROWS);
            bulk_commit_group();
          }
        }
      } else {
        // lane = query row, registers = its d features.  Each 32-feature panel row is 128
        // bytes, stored with the 128-byte swizzle (16-byte chunk j of row q at j ^ (q & 7))
        // so that eight consecutive rows hit eight different bank groups; the tensor map
        // uses the same swizzle for the bulk reduction.
        const int qr = lane_base + lane;
        if (warp == 8 && lane == 0) bulk_wait_group_read0();
        named_barrier_sync(1, 128);
        uint8_t* stg = smem + C::O_STG;
#pragma unroll
        for (int pn = 0; pn < D / 32; ++pn)
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int e = pn * 32 + j * 4;
            const float m = p.dq_mul;
            *reinterpret_cast<float4*>(stg + pn * C::STG_PANEL_BYTES + sw128_offset(qr, j)) =
                make_float4(__uint_as_float(r[e / 32][e % 32]) * m, __uint_as_float(r[e / 32][e % 32 + 1]) * m,
                            __uint_as_float(r[e / 32][e % 32 + 2]) * m, __uint_as_float(r[e / 32][e % 32 + 3]) * m);
          }
        fence_proxy_async_smem();
        named_barrier_sync(1, 128);
        if (warp == 8 && lane == 0) {
          for (int pn = 0; pn < D / 32; ++pn)
            tma_reduce_add_3d(&tmDQ, sbase + C::O_STG + pn * C::STG_PANEL_BYTES, pn * 32, h, seq_start + q0);
          bulk_commit_group();
        }
      }
    }
    }
  }

  if (warp == 8 && lane == 0) bulk_wait_group0();   // bulk reductions complete
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// D_i = sum_c dO_ic O_ic (fp32, from the stored bf16 O) and zero the dQ accumulator.
// Each group of D/8 threads handles one (token, head) row with 16-byte loads.
template <int D>
__global__ void __launch_bounds__(256) bwd_preprocess(const __nv_bfloat16* __restrict__ o,
                                                      const __nv_bfloat16* __restrict__ dout, int64_t rows, int hq,
                                                      int total_tokens, float* __restrict__ dd,
                                                      float* __restrict__ dq_acc, int zero_acc,
                                                      int* __restrict__ item_counter) {
  constexpr int TPR = D / 8;   // threads per row
  if (blockIdx.x == 0 && threadIdx.x == 0) *item_counter = 0;   // the main kernel's work-item counter
  const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t nthreads = (int64_t)gridDim.x * blockDim.x;
  // The loop condition is uniform over each warp (it tests the warp's first row), so the
  // row-group shuffles below always run with all 32 lanes present.
  const int64_t lane = threadIdx.x & 31;
  for (int64_t base = tid; (base - lane) / TPR < rows; base += nthreads) {
    const int64_t row = base / TPR;          // row = token * hq + head
    const int part = (int)(base % TPR);
    float acc = 0.f;
    if (row < rows) {
      const uint4 a = *reinterpret_cast<const uint4*>(o + row * D + part * 8);
      const uint4 bb = *reinterpret_cast<const uint4*>(dout + row * D + part * 8);
      const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
      const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&bb);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 x = __bfloat1622float2(a2[e]);
        const float2 y = __bfloat1622float2(b2[e]);
        acc = fmaf(x.x, y.x, acc);
        acc = fmaf(x.y, y.y, acc);
      }
      if (zero_acc) {
        float4* z = reinterpret_cast<float4*>(dq_acc + row * D + part * 8);
        z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
        z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
#pragma unroll
    for (int off = TPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (row < rows && part == 0) {
      const int64_t t = row / hq;
      const int h = (int)(row % hq);
      dd[(int64_t)h * total_tokens + t] = acc;
    }
  }
}

// dQ = bf16(scale * accumulator), 8 elements per thread.
__global__ void __launch_bounds__(256) bwd_dq_convert(const float* __restrict__ acc, int64_t n8, float scale,
                                                      __nv_bfloat16* __restrict__ dq) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += (int64_t)gridDim.x * blockDim.x) {
    const float4 a = reinterpret_cast<const float4*>(acc)[2 * i];
    const float4 b = reinterpret_cast<const float4*>(acc)[2 * i + 1];
    uint4 w;
    w.x = pack_bf16x2(a.x * scale, a.y * scale);
    w.y = pack_bf16x2(a.z * scale, a.w * scale);
    w.z = pack_bf16x2(b.x * scale, b.y * scale);
    w.w = pack_bf16x2(b.z * scale, b.w * scale);
    reinterpret_cast<uint4*>(dq)[i] = w;
  }
}

int sm_count() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  }
  return n;
}

// Accumulate mode (acc != nullptr): dq_acc, dk_acc, dv_acc are the caller's float32
// tensors; the gradients are added into them and nothing is written as bf16.
struct BwdAccum {
  float* dq_acc;
  float* dk_acc;
  float* dv_acc;
};

template <int D>
cudaError_t launch_bwd_d(const Problem& pb, const void* q, const void* k, const void* v, const void* o,
                         const void* dout, const float* lse, void* dq, void* dk, void* dv, void* workspace,
                         const BwdAccum* acc, cudaStream_t stream) {
  using C = BwdCfg<D>;
  const size_t T = (size_t)pb.total_tokens;
  float* dd = static_cast<float*>(workspace);
  const size_t dbytes = ((size_t)pb.hq * T * sizeof(float) + 255) & ~(size_t)255;
  float* dq_acc = acc ? acc->dq_acc : reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + dbytes);
  int* item_counter = reinterpret_cast<int*>(static_cast<uint8_t*>(workspace) + dbytes +
                                             T * (size_t)pb.hq * (size_t)D * sizeof(float));
  const int64_t rows = (int64_t)T * pb.hq;
  {
    const int64_t threads = rows * (D / 8);
    const int blocks = (int)std::min<int64_t>((threads + 255) / 256, (int64_t)sm_count() * 16);
    LaunchScope scope(K_BWD_PREPROCESS, stream);
    bwd_preprocess<D><<<blocks, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(o),
                                                   static_cast<const __nv_bfloat16*>(dout), rows, pb.hq,
                                                   pb.total_tokens, dd, dq_acc, acc ? 0 : 1, item_counter);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  alignas(64) CUtensorMap tq, tk, tv, tdo, tdq;
  if (!encode_tma_3d_f32(&tdq, dq_acc, D, pb.hq, pb.total_tokens, C::DQT ? D : 32, C::STG_ROWS) ||
      !encode_tma_3d(&tq, q, D, pb.hq, pb.total_tokens, C::PANEL, C::BM) ||
      !encode_tma_3d(&tdo, dout, D, pb.hq, pb.total_tokens, C::PANEL, C::BM) ||
      !encode_tma_3d(&tk, k, D, pb.hkv, pb.total_tokens, C::PANEL, kKeys) ||
      !encode_tma_3d(&tv, v, D, pb.hkv, pb.total_tokens, C::PANEL, kKeys))
    return cudaErrorInvalidValue;
  BwdParams p;
  p.cu_seqlens = pb.cu_seqlens;
  p.seqlen = pb.seqlen;
  p.max_seqlen = pb.max_seqlen;
  p.total_tokens = pb.total_tokens;
  p.hq = pb.hq;
  p.hkv = pb.hkv;
  p.scale = pb.scale;
  p.scale_log2 = pb.scale * kLog2e;
  p.causal = pb.causal;
  p.lse = lse;
  p.dd = dd;
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.batch = pb.batch;
  p.n_kt = (pb.max_seqlen + kKeys - 1) / kKeys;
  const int64_t items = (int64_t)p.n_kt * pb.hkv * pb.batch;
  if (items > INT32_MAX) return cudaErrorInvalidValue;
  p.n_items = (int)items;
  // Causal order: heaviest-first in groups of heads whose Q and dO together stay within
  // ~32 MB of L2.  Measured on B200 it pays at d = 128 (64-query steps: an item is twice as
  // many steps, long enough to hide its boundary) and loses at d <= 64, where the key
  // tiles of one head in turn are faster.
  p.heads_per_group = -1;
  if (pb.causal && D == 128) {
    const int64_t head_bytes = (int64_t)(pb.hq / pb.hkv) * pb.max_seqlen * D * 2 * 2;
    const int64_t pairs = (int64_t)pb.hkv * pb.batch;
    p.heads_per_group = (int)std::max<int64_t>(1, std::min<int64_t>(pairs, (32ll << 20) / std::max<int64_t>(head_bytes, 1)));
  }
  p.item_counter = item_counter;
  p.dq_acc = dq_acc;
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);
  p.accumulate = acc ? 1 : 0;
  p.dq_mul = acc ? pb.scale : 1.f;
  p.dk_acc = acc ? acc->dk_acc : nullptr;
  p.dv_acc = acc ? acc->dv_acc : nullptr;
  cudaError_t e = cudaFuncSetAttribute(bwd_bf16_sm100<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  // persistent: one CTA per SM (shared memory allows no more) walking its item list
  const int grid = (int)std::min<int64_t>(items, sm_count());
  {
    LaunchScope scope(K_BWD_BF16, stream);
    bwd_bf16_sm100<D><<<grid, kThreads, C::SMEM_BYTES, stream>>>(tq, tk, tv, tdo, tdq, p);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) return e;
  if (acc) return cudaSuccess;   // the caller's accumulator stays float32
  const int64_t n8 = rows * D / 8;
  const int blocks = (int)std::min<int64_t>((n8 + 255) / 256, (int64_t)sm_count() * 16);
  LaunchScope scope(K_BWD_DQ_CONVERT, stream);
  bwd_dq_convert<<<blocks, 256, 0, stream>>>(dq_acc, n8, pb.scale, static_cast<__nv_bfloat16*>(dq));
  return cudaGetLastError();
}

}  // namespace

size_t bwd_bf16_workspace_bytes(const Problem& pb) {
  const size_t T = (size_t)pb.total_tokens;
  const size_t dbytes = ((size_t)pb.hq * T * sizeof(float) + 255) & ~(size_t)255;   // D [hq, T]
  const size_t qacc = T * (size_t)pb.hq * (size_t)pb.d * sizeof(float);             // dQ accumulator
  return dbytes + qacc + 256;                                                       // + item counter
}

cudaError_t launch_bwd_bf16(const Problem& pb, const void* q, const void* k, const void* v, const void* o,
                            const void* dout, const float* lse, void* dq, void* dk, void* dv, void* workspace,
                            cudaStream_t stream) {
  if (pb.total_tokens == 0 || pb.batch == 0 || pb.max_seqlen == 0) return cudaSuccess;
  switch (pb.d) {
    case 32: return launch_bwd_d<32>(pb, q, k, v, o, dout, lse, dq, dk, dv, workspace, nullptr, stream);
    case 64: return launch_bwd_d<64>(pb, q, k, v, o, dout, lse, dq, dk, dv, workspace, nullptr, stream);
    case 128: return launch_bwd_d<128>(pb, q, k, v, o, dout, lse, dq, dk, dv, workspace, nullptr, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_bwd_bf16_accumulate(const Problem& pb, const void* q, const void* k, const void* v, const void* o,
                                       const void* dout, const float* lse, float* dq_acc, float* dk_acc,
                                       float* dv_acc, void* workspace, cudaStream_t stream) {
  if (pb.total_tokens == 0 || pb.batch == 0 || pb.max_seqlen == 0) return cudaSuccess;
  const BwdAccum acc{dq_acc, dk_acc, dv_acc};
  switch (pb.d) {
    case 32: return launch_bwd_d<32>(pb, q, k, v, o, dout, lse, nullptr, nullptr, nullptr, workspace, &acc, stream);
    case 64: return launch_bwd_d<64>(pb, q, k, v, o, dout, lse, nullptr, nullptr, nullptr, workspace, &acc, stream);
    case 128: return launch_bwd_d<128>(pb, q, k, v, o, dout, lse, nullptr, nullptr, nullptr, workspace, &acc, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace attn
