// fwd_sm100.cu -- exact attention forward for sm_100a: TMA + tcgen05 + TMEM.
//
// What it computes: O = softmax(scale * Q K^T [+ causal mask]) V and the per-row
// LSE = m + ln l, for every (sequence, query head) ("FlashAttention 与高效注意力内核"
// tutorial, sections 标准注意力三步 and 前向).
//
// How (sections 分块, Online Softmax 技巧 and 伪代码骨架 of the same tutorial; FA2's
// query-outer loop order from the "Flash-Attention" concept page, 核心思想): a work item
// is two 128-row query tiles of one head; the item streams the sequence's 128-key K/V
// tiles through shared memory once.  Per key tile and query tile t:
//     S_t   = Q_t K_j^T                  tcgen05 MMA, A and B from swizzled SMEM, fp32 in TMEM
//     m_new = max(m_old, rowmax(S_t))    one query row per thread, no shuffles
//     P_t   = exp2(S_t * scale*log2e - m_new), l = l * exp2(m_old - m_new) + rowsum(P_t)
//     O_t   = exp2(m_old - m_new) * O_t + P_t V_j
// with P_t stored as bf16 into the TMEM columns that held S_t and fed to the PV MMA
// straight from TMEM.  The running O_t never leaves TMEM until the end, where it is
// divided by l and written once with LSE (the tutorial's 前向: only O and the row
// statistics reach HBM).
//
// Rescale skipping: m_new only moves when the tile max exceeds the running max by more
// than 8 (in log2 units).  Otherwise the old max keeps being used, so P entries stay
// <= 2^8 and O, l are left as they are; the final O / l and LSE use that same max
// consistently, so the result is exact up to rounding.  (The concept page lists this
// "conditional rescaling" among the Blackwell techniques, 已知局限.)
//
// Persistent schedule: one CTA per SM claims work items from a global counter in a fixed
// order -- heaviest first under the causal mask, within groups of heads whose K/V fit in
// L2; pairs of one head adjacent otherwise (their K/V stream is shared through L2), with
// a last wave that would leave most SMs idle split into single-tile items.  All pipelines
// run across items: each Q tile buffer reloads as soon as its own last QK^T is done, the
// next item's first QK^T MMAs overlap the current item's epilogue, and the K/V ring never
// drains.  Under the causal mask a query tile only visits key tiles it can see, so the
// lower tile of an item skips the last key tile.
//
// Warp roles (320 threads):
//   warps 0-3  softmax + correction + epilogue for query tile 0 (TMEM lanes 0..127)
//   warps 4-7  the same for query tile 1
//   warp  8    TMA producer: Q tiles per item, K_j / V_j into a STAGES-deep ring
//   warp  9    MMA issuer (one thread): S0, S1, then PV0, S0', PV1, S1', ... so the tensor
//              core works on one tile while the other tile's softmax runs.
// TMEM (512 columns x 128 lanes, fp32): S0 [0,128) S1 [128,256) O0 [256,256+d) O1 after.
#include <algorithm>

#include "kernels.h"
#include "sm100.cuh"

namespace attn {

namespace {

constexpr int kRows = 128;                 // query rows per tile == TMEM lanes
constexpr int kKeys = 128;                 // keys per K/V tile
constexpr float kRescaleSkip = 8.0f;       // log2 units, see file comment
// Pairs of exponentials computed on the FMA pipe in unmasked tiles: bit (c % 8) of this
// mask selects pair c (2 of every 8 pairs, 25%, the best of 0 / 25 / 37.5 / 50% measured
// on B200), balancing the special-function unit against the FMA pipe.
constexpr uint32_t kEmuPairs = 0x22u;
// The same for the FP8 forward, whose products take half the tensor-core time.
constexpr uint32_t kEmuPairsFp8 = 0x22u;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kThreads = 320;
constexpr int kItemSlots = 4;  // ring of work-item indices the producer hands to the other roles

// FP8: Q, K and V^T (per-head transposed V) are e4m3 tiles and both products run as
// kind::f8f6f4 with 32-element K steps; P goes to TMEM as four e4m3 per column.  A Q / K
// row is d bytes (128: one 128-byte swizzle span; 64: the 64-byte swizzle), a V^T row is
// 128 keys = 128 bytes whatever d is.
template <int D, bool FP8 = false>
struct FwdCfg {
  static constexpr int ELEM = FP8 ? 1 : 2;         // bytes per Q/K/V element
  static constexpr int SW = D * ELEM >= 128 ? 128 : 64;   // swizzle span == SMEM row pitch (bytes)
  static constexpr int PANEL = SW / ELEM;          // elements per panel row
  static constexpr int NPANEL = D / PANEL;         // panels per tile
  static constexpr int PANEL_BYTES = kRows * SW;   // one panel of a 128-row tile
  static constexpr int TILE_BYTES = kRows * D * ELEM;
  static constexpr int STAGES = FP8 ? 4 : (D == 128 ? 2 : (D == 64 ? 3 : 4));
  static constexpr uint32_t SWZ = SW == 128 ? 2u : 4u;   // descriptor swizzle code
  static constexpr int SBO = 8 * SW;               // bytes between 8-row swizzle atoms
  // FP8 V^T tile: d rows of 128 keys, always the 128-byte swizzle
  static constexpr uint32_t VT_SWZ = 2u;
  static constexpr int VT_SBO = 1024;
  static constexpr int KSTEPS_PER_PANEL = SW / 32; // 32-byte K steps inside one panel
  static constexpr int S_KSTEPS = D * ELEM / 32;   // K steps of Q K^T
  static constexpr int PV_KSTEPS = kKeys * ELEM / 32;   // K steps of P V (8 P columns each)
  // barrier slots
  static constexpr int B_QFULL = 0;                  // 2: one per query tile
  static constexpr int B_QEMPTY = 2;                 // 2
  static constexpr int B_KFULL = 4;
  static constexpr int B_VFULL = B_KFULL + STAGES;
  static constexpr int B_KEMPTY = B_VFULL + STAGES;
  static constexpr int B_VEMPTY = B_KEMPTY + STAGES;
  static constexpr int B_SFULL = B_VEMPTY + STAGES;  // 2
  static constexpr int B_PFULL = B_SFULL + 2;        // 2
  static constexpr int B_OFINAL = B_PFULL + 2;       // 2
  static constexpr int B_OFREE = B_OFINAL + 2;       // 2
  static constexpr int B_IFULL = B_OFREE + 2;        // kItemSlots: item index written
  static constexpr int B_IEMPTY = B_IFULL + kItemSlots;   // kItemSlots: read by MMA + softmax warps
  static constexpr int B_DRAIN = B_IEMPTY + kItemSlots;   // the MMA issuer's completion at exit
  static constexpr int NBARS = B_DRAIN + 1;
  // Epilogue staging: each softmax warp turns its 32 O rows into coalesced stores through a
  // 32-row slice of STG_ROWB bytes per row (half a row per pass at d = 128).
  static constexpr int STG_ROWB = D * 2 < 128 ? D * 2 : 128;
  static constexpr int STG_PASSES = D * 2 / STG_ROWB;
  static constexpr int STG_WARP_BYTES = 32 * STG_ROWB;
  static constexpr int O_STG = (2 + 2 * STAGES) * TILE_BYTES;
  static constexpr int DATA_BYTES = O_STG + 8 * STG_WARP_BYTES;
  // after the barriers: TMEM address, abort flag, the item-index ring
  static constexpr int SMEM_BYTES = 1024 + DATA_BYTES + NBARS * 8 + 8 + 4 * kItemSlots;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

struct FwdParams {
  const int32_t* cu_seqlens;
  int32_t seqlen, max_seqlen, total_tokens, hq, hkv, batch;
  int32_t n_pairs, n_items;
  int32_t n_full;    // items [0, n_full) are two-tile items; the rest single query tiles
  float scale_log2;  // scale * log2(e), rounded to fp32
  double lse_skew;   // scale_log2 * ln 2 - scale, in double: the rounding of scale_log2
  int32_t causal;
  __nv_bfloat16* o;
  float* lse;
  const float* descale_q;    // FP8: per query head
  const float* descale_k;    // FP8: per kv head
  const float* descale_v;    // FP8: per kv head
  int32_t heads_per_group;   // causal order: (head, sequence) pairs whose K / V fit in L2
  int* item_counter;         // next unclaimed item (zeroed before the launch)
};

// One work item: two query tiles of one head of one sequence.
struct Item {
  int h, b, seq_start, len, q0;
  int n[2];    // key tiles each query tile visits (0: the tile is past the sequence)
  int nkv;     // key tiles loaded for the item, max(n[0], n[1])
};

// Work item number idx.  The CTAs are persistent (one per SM) and claim items in this
// order from a global counter, so each takes the next one as soon as it is free.  Causal:
// heaviest first (the last query tiles see the most keys) within groups of
// (head, sequence) pairs whose K / V fit in about 32 MB of L2, so that the items in flight
// share what they stream, and lighter items fill in at the end.  Otherwise the pairs of
// one head are consecutive (their K / V stream is shared through L2), and when the last
// wave of two-tile items would leave more than half of the SMs idle, the pairs of that
// wave are split into single-tile items (items n_full, n_full + 1 are the two tiles of
// pair n_full, and so on), which fill twice as many SMs.
__device__ __forceinline__ Item item_from(const FwdParams& p, int idx) {
  Item it;
  if (idx < 0 || idx >= p.n_items) {
    it.h = it.b = it.seq_start = it.len = it.q0 = 0;
    it.n[0] = it.n[1] = it.nkv = 0;
    return it;
  }
  int pair;
  int single = 0;   // 0: both tiles of the pair; 1 / 2: only its first / second tile
  if (p.causal) {
    const int pairs = p.hq * p.batch;
    const int per_grp = p.n_pairs * p.heads_per_group;
    const int grp = idx / per_grp, rem = idx % per_grp;
    const int ng = min(p.heads_per_group, pairs - grp * p.heads_per_group);
    pair = p.n_pairs - 1 - rem / ng;
    const int r = grp * p.heads_per_group + rem % ng;
    it.h = r % p.hq;
    it.b = r / p.hq;
  } else {
    int pr = idx;
    if (idx >= p.n_full) {
      pr = p.n_full + (idx - p.n_full) / 2;
      single = 1 + ((idx - p.n_full) & 1);
    }
    pair = pr % p.n_pairs;
    const int t = pr / p.n_pairs;
    it.h = t % p.hq;
    it.b = t / p.hq;
  }
  it.seq_start = p.cu_seqlens ? p.cu_seqlens[it.b] : it.b * p.seqlen;
  it.len = p.cu_seqlens ? p.cu_seqlens[it.b + 1] - it.seq_start : p.seqlen;
  it.q0 = pair * 2 * kRows + (single == 2 ? kRows : 0);
  for (int t = 0; t < 2; ++t) {
    const int r0 = it.q0 + t * kRows;
    if (r0 >= it.len || (single && t == 1)) {
      it.n[t] = 0;
    } else {
      const int kv_end = p.causal ? min(it.len, r0 + kRows) : it.len;
      it.n[t] = (kv_end + kKeys - 1) / kKeys;
    }
  }
  it.nkv = max(it.n[0], it.n[1]);
  return it;
}

template <int D, bool FP8>
__device__ __forceinline__ void fwd_body(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                                         const FwdParams& p) {
  using C = FwdCfg<D, FP8>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);   // 1024-aligned (swizzle atoms)
  const uint32_t sQ = smem_u32(smem);
  const uint32_t sK = sQ + 2 * C::TILE_BYTES;
  const uint32_t sV = sK + C::STAGES * C::TILE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::DATA_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NBARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* s_items = reinterpret_cast<volatile int*>(tmem_slot + 2);
  auto bar = [&](int i) { return smem_u32(bars + i); };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // The producer claims items and hands their indices to the MMA issuer and the softmax
  // warps through the s_items ring, so all roles walk the same items in the same order.
  // next_item(k) returns the k-th claimed index (-1 after a failed wait); an index
  // >= n_items ends the walk.
  auto next_item = [&](int k) -> int {
    const int slot = k % kItemSlots;
    if (!mbar_wait(bar(C::B_IFULL + slot), (k / kItemSlots) & 1, abort_flag)) return -1;
    const int idx = s_items[slot];
    __syncwarp(__activemask());
    if ((threadIdx.x & 31) == __ffs(__activemask()) - 1) mbar_arrive(bar(C::B_IEMPTY + slot));
    return idx;
  };

  if (threadIdx.x == 0) {
    // sequences longer than max_seqlen would not be covered by the item list
    if (blockIdx.x == 0)
      for (int b = 0; b < p.batch; ++b) {
        const int len = p.cu_seqlens ? p.cu_seqlens[b + 1] - p.cu_seqlens[b] : p.seqlen;
        if (len > p.max_seqlen) report_error(ATTN_DEVERR_SEQLEN);
      }
    for (int i = 0; i < C::NBARS; ++i) {
      // P-ready and O-free are arrived on once per softmax warp (after __syncwarp)
      const bool per_warp = (i == C::B_PFULL || i == C::B_PFULL + 1 || i == C::B_OFREE || i == C::B_OFREE + 1);
      // an item slot is read by the MMA issuer and the 8 softmax warps
      const bool slot_read = i >= C::B_IEMPTY && i < C::B_IEMPTY + kItemSlots;
      mbar_init(bar(i), slot_read ? 9u : (per_warp ? 4u : 1u));
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 8) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      uint32_t kv = 0;            // K/V tiles so far
      uint32_t qc[2] = {0, 0};    // loads of each query tile buffer so far
      uint32_t kc = 0, vc = 0;    // K and V loads issued
      bool ok = true;
      for (int k = 0; ok; ++k) {
        // claim the next item and hand its index to the other roles
        const int slot = k % kItemSlots;
        if (!mbar_wait(bar(C::B_IEMPTY + slot), ((k / kItemSlots) & 1) ^ 1, abort_flag)) break;
        const int idx = atomicAdd(p.item_counter, 1);
        s_items[slot] = idx;
        mbar_arrive(bar(C::B_IFULL + slot));
        if (idx >= p.n_items) break;
        const Item it = item_from(p, idx);
        if (it.nkv == 0) continue;
        const int hk = it.h / (p.hq / p.hkv);
        // Each query tile buffer reloads as soon as its own last QK^T of the previous item
        // is done (under the causal mask tile 0's comes a key tile earlier), and tile 1
        // after the item's first K tile, so the item's first product can start while the
        // previous item's tile 1 still runs.
        auto load_q = [&](int t) -> bool {
          if (it.n[t] == 0) return true;
          if (!mbar_wait(bar(C::B_QEMPTY + t), (qc[t] & 1) ^ 1, abort_flag)) return false;
          mbar_arrive_expect_tx(bar(C::B_QFULL + t), C::TILE_BYTES);
          for (int pn = 0; pn < C::NPANEL; ++pn)
            tma_load_3d(sQ + t * C::TILE_BYTES + pn * C::PANEL_BYTES, &tmQ, bar(C::B_QFULL + t), pn * C::PANEL, it.h,
                        it.seq_start + it.q0 + t * kRows);
          ++qc[t];
          return true;
        };
        if (!load_q(0)) break;
        for (int j = 0; j < it.nkv; ++j, ++kv) {
          const int s = kv % C::STAGES;
          const uint32_t ph = (kv / C::STAGES) & 1;
          if (!mbar_wait(bar(C::B_KEMPTY + s), ph ^ 1, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(bar(C::B_KFULL + s), C::TILE_BYTES);
          for (int pn = 0; pn < C::NPANEL; ++pn)
            tma_load_3d(sK + s * C::TILE_BYTES + pn * C::PANEL_BYTES, &tmK, bar(C::B_KFULL + s), pn * C::PANEL, hk,
                        it.seq_start + j * kKeys);
          ++kc;
          if (j == 0 && !load_q(1)) { ok = false; break; }
          if (!mbar_wait(bar(C::B_VEMPTY + s), ph ^ 1, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(bar(C::B_VFULL + s), C::TILE_BYTES);
          ++vc;
          if constexpr (FP8) {
            // V^T [batch * hkv][d][padded seqlen]: a (128 keys) x (d rows) box, keys
            // contiguous (K-major B); the key coordinate is a multiple of 128
            tma_load_3d(sV + s * C::TILE_BYTES, &tmV, bar(C::B_VFULL + s), j * kKeys, 0, it.b * p.hkv + hk);
          } else {
            for (int pn = 0; pn < C::NPANEL; ++pn)
              tma_load_3d(sV + s * C::TILE_BYTES + pn * C::PANEL_BYTES, &tmV, bar(C::B_VFULL + s), pn * C::PANEL, hk,
                          it.seq_start + j * kKeys);
          }
        }
      }
      // Every load issued here lands before the CTA releases its memory, also when another
      // role gave up waiting: only the last load of each stage can still be in flight (a
      // stage is reloaded only after its previous contents were consumed).
      for (uint32_t i = kc > (uint32_t)C::STAGES ? kc - C::STAGES : 0; i < kc; ++i)
        mbar_wait_drain(bar(C::B_KFULL + i % C::STAGES), (i / C::STAGES) & 1);
      for (uint32_t i = vc > (uint32_t)C::STAGES ? vc - C::STAGES : 0; i < vc; ++i)
        mbar_wait_drain(bar(C::B_VFULL + i % C::STAGES), (i / C::STAGES) & 1);
      for (int t = 0; t < 2; ++t)
        if (qc[t] > 0) mbar_wait_drain(bar(C::B_QFULL + t), (qc[t] - 1) & 1);
    }
  } else if (warp == 9) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      // Q, K both K-major; V is MN-major in bf16 (d contiguous), V^T K-major in FP8
      const uint32_t idesc_qk = FP8 ? idesc_e4m3_f32(kRows, kKeys, false, false)
                                    : idesc_bf16_f32(kRows, kKeys, false, false);
      const uint32_t idesc_pv = FP8 ? idesc_e4m3_f32(kRows, D, false, false) : idesc_bf16_f32(kRows, D, false, true);
      // Operand descriptors: bases computed once, advanced by compile-time offsets per
      // MMA (and by the tile/stage index per call), so one MMA issues in a few
      // instructions -- this single thread's issue rate bounds the tensor core.
      const uint64_t q_desc = smem_desc(sQ, 16, C::SBO, C::SWZ);
      const uint64_t k_desc = smem_desc(sK, 16, C::SBO, C::SWZ);
      const uint64_t v_desc = FP8 ? smem_desc(sV, 16, C::VT_SBO, C::VT_SWZ)
                                  : smem_desc(sV, C::PANEL_BYTES, C::SBO, C::SWZ);
      auto issue_qk = [&](int t, int s) {
        const uint32_t d_tmem = tmem + t * kKeys;
        const uint64_t a0 = desc_advance(q_desc, (uint32_t)t * C::TILE_BYTES);
        const uint64_t b0 = desc_advance(k_desc, (uint32_t)s * C::TILE_BYTES);
#pragma unroll
        for (int kk = 0; kk < C::S_KSTEPS; ++kk) {
          const uint32_t off = (kk / C::KSTEPS_PER_PANEL) * C::PANEL_BYTES + (kk % C::KSTEPS_PER_PANEL) * 32;
          if constexpr (FP8)
            mma_ss_f8(d_tmem, desc_advance(a0, off), desc_advance(b0, off), idesc_qk, kk > 0 ? 1u : 0u);
          else
            mma_ss(d_tmem, desc_advance(a0, off), desc_advance(b0, off), idesc_qk, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int t, int s, bool accumulate) {
        const uint32_t d_tmem = tmem + 2 * kKeys + t * D;
        const uint64_t b0 = desc_advance(v_desc, (uint32_t)s * C::TILE_BYTES);
#pragma unroll
        for (int kk = 0; kk < C::PV_KSTEPS; ++kk) {
          const uint32_t a_tmem = tmem + t * kKeys + kk * 8;   // 8 packed columns: 16 bf16 / 32 e4m3 keys
          if constexpr (FP8)
            mma_ts_f8(d_tmem, a_tmem, desc_advance(b0, kk * 32), idesc_pv, (accumulate || kk > 0) ? 1u : 0u);
          else
            mma_ts(d_tmem, a_tmem, desc_advance(b0, kk * 16 * C::SW), idesc_pv, (accumulate || kk > 0) ? 1u : 0u);
        }
      };
      uint32_t kv = 0;
      uint32_t qm[2] = {0, 0};   // loads of each query tile buffer consumed
      uint32_t pc[2] = {0, 0};   // P_t tiles consumed
      uint32_t om[2] = {0, 0};   // items started per query tile (for the O-free handshake)
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int idx = next_item(k);
        if (idx < 0 || idx >= p.n_items) break;
        const Item it = item_from(p, idx);
        if (it.nkv == 0) continue;
        int rem[2] = {it.n[0], it.n[1]};   // QK^T MMAs still to issue per tile; Q_t is free after its last
        const int s0 = kv % C::STAGES;
        ok = mbar_wait(bar(C::B_KFULL + s0), (kv / C::STAGES) & 1, abort_flag);
        for (int t = 0; ok && t < 2; ++t)
          if (it.n[t] > 0) {
            if (!mbar_wait(bar(C::B_QFULL + t), qm[t] & 1, abort_flag)) { ok = false; break; }
            ++qm[t];
            tc_fence_after();
            issue_qk(t, s0);
            mma_commit(bar(C::B_SFULL + t));
            if (--rem[t] == 0) mma_commit(bar(C::B_QEMPTY + t));
          }
        if (!ok) break;
        mma_commit(bar(C::B_KEMPTY + s0));
        // The V and K stages and the other tile's P are checked with mbar_test while the
        // preceding MMAs issue (mbar_wait only if they had not completed then): a check that
        // waits for its own shared-memory round trip leaves the tensor pipe's short queue idle.
        bool v_ready = false;   // V tile of step j seen complete during step j - 1
        for (int j = 0; ok && j < it.nkv; ++j) {
          const uint32_t c = kv + j;
          const int s = c % C::STAGES;
          if (!v_ready && !mbar_wait(bar(C::B_VFULL + s), (c / C::STAGES) & 1, abort_flag)) { ok = false; break; }
          bool k_next = false;
          const int s1 = (c + 1) % C::STAGES;
          const bool k_ready = j + 1 < it.nkv && mbar_test(bar(C::B_KFULL + s1), ((c + 1) / C::STAGES) & 1);
          bool p_ready = false;   // this tile's P seen complete while the other tile's products issued
          for (int t = 0; t < 2; ++t) {
            if (j >= it.n[t]) continue;
            if (!p_ready && !mbar_wait(bar(C::B_PFULL + t), pc[t] & 1, abort_flag)) { ok = false; break; }
            ++pc[t];
            if (j == 0) {   // O_t of the previous item has been read out
              if (!mbar_wait(bar(C::B_OFREE + t), (om[t] & 1) ^ 1, abort_flag)) { ok = false; break; }
              ++om[t];
            }
            tc_fence_after();
            issue_pv(t, s, j > 0);
            p_ready = t == 0 && j < it.n[1] && mbar_test(bar(C::B_PFULL + 1), pc[1] & 1);
            if (j + 1 < it.n[t]) {
              if (!k_next) {
                if (!k_ready && !mbar_wait(bar(C::B_KFULL + s1), ((c + 1) / C::STAGES) & 1, abort_flag)) {
                  ok = false;
                  break;
                }
                tc_fence_after();
                k_next = true;
              }
              issue_qk(t, s1);
              mma_commit(bar(C::B_SFULL + t));
              if (--rem[t] == 0) mma_commit(bar(C::B_QEMPTY + t));
            } else {
              mma_commit(bar(C::B_OFINAL + t));
            }
          }
          if (!ok) break;
          v_ready = j + 1 < it.nkv && mbar_test(bar(C::B_VFULL + s1), ((c + 1) / C::STAGES) & 1);
          mma_commit(bar(C::B_VEMPTY + s));
          if (k_next) mma_commit(bar(C::B_KEMPTY + s1));
        }
        kv += it.nkv;
      }
      // every MMA issued here has completed before the CTA frees Tensor Memory
      mma_commit(bar(C::B_DRAIN));
      mbar_wait_drain(bar(C::B_DRAIN), 0);
    }
  } else {
    // ---------------- softmax / correction / epilogue (one query row per thread) ---------
    const int t = warp >> 2;                        // query tile of this warpgroup
    const int lane_base = (warp & 3) * 32;          // TMEM lanes this warp may touch
    const uint32_t tS = tmem + ((uint32_t)lane_base << 16) + t * kKeys;
    const uint32_t tO = tmem + ((uint32_t)lane_base << 16) + 2 * kKeys + t * D;
    const float sl2_base = p.scale_log2;
    uint32_t sc = 0, oc = 0;   // S_t tiles and items consumed by this warpgroup
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int idx = next_item(k);
      if (idx < 0 || idx >= p.n_items) break;
      const Item it = item_from(p, idx);
      const int n_t = it.n[t];
      if (n_t == 0) continue;
      const int qi = it.q0 + t * kRows + lane_base + lane;   // query index inside the sequence
      // FP8: the e4m3 products carry the per-head scales of Q and K
      const int hk = it.h / (p.hq / p.hkv);
      const float sl2 = FP8 ? sl2_base * p.descale_q[it.h] * p.descale_k[hk] : sl2_base;
      float m_used = -INFINITY;   // running max in log2 units (possibly stale by < 8)
      float mx_used = 0.f;        // the raw score maximum that m_used was formed from
      float l = 0.f;              // running sum of exp2(x - m_used)
      for (int j = 0; j < n_t; ++j) {
        if (!mbar_wait(bar(C::B_SFULL + t), sc & 1, abort_flag)) { ok = false; break; }
        ++sc;
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
        // mask: key kbase + c is visible iff it is inside the sequence and, when causal,
        // not after this query.
        const int kbase = j * kKeys;
        int lim = it.len - 1 - kbase;
        if (p.causal) lim = min(lim, qi - kbase);
        const bool masked = lim < kKeys - 1;
        if (masked) {
#pragma unroll
          for (int c = 0; c < kKeys; ++c)
            if (c > lim) s[c] = -INFINITY;
        }
        // Row max over 8 independent partial maxima (short dependency chains).
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
        // P as bf16 pairs (64 columns) or, FP8, e4m3 quads (32 columns); key 2c, 2c+1 -> pair c
        uint32_t pk[64];
        auto put_p = [&](uint32_t (&w)[64], int c, float p0, float p1) {
          if constexpr (FP8) {
            const uint32_t h = pack_e4m3x2(p0, p1);
            if (c & 1) w[c >> 1] |= h << 16;
            else w[c >> 1] = h;
          } else {
            w[c] = pack_bf16x2(p0, p1);
          }
        };
        const uint64_t sl2x2 = f2(sl2, sl2);
        const uint64_t negm = f2(-m_sub, -m_sub);
        uint64_t sum2[4] = {f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f)};   // 8 partial sums
        if (masked) {
          // hidden keys must come out as exact zeros: special-function unit only
#pragma unroll
          for (int c = 0; c < 64; ++c) {
            float x0, x1;
            f2_split(fma2(f2(s[2 * c], s[2 * c + 1]), sl2x2, negm), x0, x1);
            const float p0 = ex2(x0), p1 = ex2(x1);
            sum2[c & 3] = add2(sum2[c & 3], f2(p0, p1));
            put_p(pk, c, p0, p1);
          }
        } else {
          // A share of the exponentials (the pairs c with bit c % 8 set in kEmuPairs) runs
          // on the FMA pipe, the rest on the special-function unit, so the two units share
          // the row's exponential work.
#pragma unroll
          for (int c = 0; c < 64; ++c) {
            const uint64_t x = fma2(f2(s[2 * c], s[2 * c + 1]), sl2x2, negm);
            float p0, p1;
            if (((FP8 ? kEmuPairsFp8 : kEmuPairs) >> (c % 8)) & 1u) {
              ex2_fma_pair(x, p0, p1);
            } else {
              float x0, x1;
              f2_split(x, x0, x1);
              p0 = ex2(x0);
              p1 = ex2(x1);
            }
            sum2[c & 3] = add2(sum2[c & 3], f2(p0, p1));
            put_p(pk, c, p0, p1);
          }
        }
        float sum_lo, sum_hi;
        f2_split(add2(add2(sum2[0], sum2[1]), add2(sum2[2], sum2[3])), sum_lo, sum_hi);
        const float rowsum = sum_lo + sum_hi;
        {
          uint32_t (&lo)[32] = *reinterpret_cast<uint32_t(*)[32]>(&pk[0]);
          tmem_st32(tS + 0, lo);
          if constexpr (!FP8) {
            uint32_t (&hi)[32] = *reinterpret_cast<uint32_t(*)[32]>(&pk[32]);
            tmem_st32(tS + 32, hi);
          }
        }
        float alpha = 1.f;
        if (m_new != m_used) {
          alpha = ex2(m_used - m_sub);   // 0 when m_used is -inf
          l = l * alpha + rowsum;
        } else {
          l += rowsum;
        }
        const bool need = (j > 0) && (m_new != m_used);
        m_used = m_new;
        if (__any_sync(0xffffffffu, need)) {
          // O_t was last written by PV_t(j-1), which completed before S_t(j) was signalled.
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t r[32];
            tmem_ld32(tO + c * 32, r);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
            tmem_st32(tO + c * 32, r);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(C::B_PFULL + t));
      }
      if (!ok) break;
      // ---------------- epilogue: O / l and LSE, then hand O_t back to the MMA ----------------
      if (!mbar_wait(bar(C::B_OFINAL + t), oc & 1, abort_flag)) { ok = false; break; }
      ++oc;
      tc_fence_after();
      const float inv_l = (l > 0.f ? 1.f / l : 0.f) * (FP8 ? p.descale_v[hk] : 1.f);
      const bool row_ok = qi < it.len;
      // O / l as bf16, written through this warp's staging slice so that each store
      // instruction covers whole 128-byte row segments (a thread-per-row store would touch
      // 32 different lines per instruction).  16-byte chunk ch of staged row r sits at
      // chunk ch ^ (r % CH), which keeps both the row-wise writes and the segment-wise reads
      // free of bank conflicts.
      constexpr int CH = C::STG_ROWB / 16;          // 16-byte chunks per staged row
      constexpr int RPI = 32 / CH;                  // rows per coalesced store instruction
      uint8_t* stg = smem + C::O_STG + warp * C::STG_WARP_BYTES;
      const int row0 = it.q0 + t * kRows + lane_base;   // query index of the warp's first row
#pragma unroll
      for (int pass = 0; pass < C::STG_PASSES; ++pass) {
        constexpr int COLS = C::STG_ROWB / 2;       // bf16 columns per pass
        uint32_t w[COLS / 2];
#pragma unroll
        for (int c = 0; c < COLS / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(tO + pass * COLS + c * 32, r);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e)
            w[c * 16 + e] = pack_bf16x2(__uint_as_float(r[2 * e]) * inv_l, __uint_as_float(r[2 * e + 1]) * inv_l);
        }
#pragma unroll
        for (int ch = 0; ch < CH; ++ch)
          *reinterpret_cast<uint4*>(stg + lane * C::STG_ROWB + ((ch ^ (lane % CH)) << 4)) =
              make_uint4(w[4 * ch], w[4 * ch + 1], w[4 * ch + 2], w[4 * ch + 3]);
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 32 / RPI; ++i) {
          const int r = i * RPI + lane / CH;
          const int ch = lane % CH;
          const uint4 v = *reinterpret_cast<const uint4*>(stg + r * C::STG_ROWB + ((ch ^ (r % CH)) << 4));
          if (row0 + r < it.len)
            *reinterpret_cast<uint4*>(p.o + ((size_t)(it.seq_start + row0 + r) * p.hq + it.h) * D + pass * COLS +
                                      ch * 8) = v;
        }
        __syncwarp();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::B_OFREE + t));
      if (row_ok) {
        // LSE = m ln 2 + ln l, combined in double from the exact fp32 values the
        // exponentials used (m_used, l), minus the first-order effect of scale_log2 being
        // rounded to fp32 (exact when one score dominates the row), then rounded once.  ln l
        // itself comes from the fp32 logf (l <= 2^8 * n, so its error is below 1e-6): a
        // double-precision log is a long software sequence on this path, which every item
        // boundary waits for.
        // the rounding of the fp32 score factor (for FP8 it includes the two descales)
        double skew = p.lse_skew;
        if constexpr (FP8)
          skew = (double)sl2 * 0.6931471805599453 -
                 ((double)p.scale_log2 * 0.6931471805599453 - p.lse_skew) * p.descale_q[it.h] * p.descale_k[hk];
        float lse = -INFINITY;
        if (l > 0.f)
          lse = (float)((double)m_used * 0.6931471805599453 + (double)logf(l) - skew * (double)mx_used);
        p.lse[(size_t)it.h * p.total_tokens + it.seq_start + qi] = lse;
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

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_bf16_sm100(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  fwd_body<D, false>(tmQ, tmK, tmV, p);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_fp8_sm100(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmVt, const FwdParams p) {
  fwd_body<D, true>(tmQ, tmK, tmVt, p);
}

int sm_count_fwd() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  }
  return n;
}

// Parameters and schedule shared by the bf16 and FP8 launches.
template <int D, bool FP8>
FwdParams fwd_params(const Problem& pb, void* o, float* lse, void* workspace) {
  FwdParams p{};
  p.cu_seqlens = pb.cu_seqlens;
  p.seqlen = pb.seqlen;
  p.max_seqlen = pb.max_seqlen;
  p.total_tokens = pb.total_tokens;
  p.hq = pb.hq;
  p.hkv = pb.hkv;
  p.batch = pb.batch;
  p.n_pairs = (pb.max_seqlen + 2 * kRows - 1) / (2 * kRows);
  // non-causal: split the pairs of a last wave that would fill at most half of the SMs
  const int64_t pairs = (int64_t)p.n_pairs * pb.hq * pb.batch;
  const int64_t ctas = sm_count_fwd();
  const int64_t rem = pairs % ctas;
  const int64_t split = (!pb.causal && 2 * rem <= ctas) ? rem : 0;
  const int64_t items = pairs + split;
  p.n_items = items > INT32_MAX ? -1 : (int)items;
  p.n_full = (int)(pairs - split);
  p.scale_log2 = pb.scale * kLog2e;
  p.lse_skew = (double)p.scale_log2 * 0.6931471805599453 - (double)pb.scale;
  p.causal = pb.causal;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  // causal order: (head, sequence) pairs whose K and V together stay within ~32 MB of L2
  const int64_t kv_bytes = (int64_t)pb.max_seqlen * D * FwdCfg<D, FP8>::ELEM * 2;
  p.heads_per_group = (int)std::max<int64_t>(
      1, std::min<int64_t>((int64_t)pb.hq * pb.batch, (32ll << 20) / std::max<int64_t>(kv_bytes, 1)));
  p.item_counter = static_cast<int*>(workspace);
  return p;
}

template <int D, bool FP8, typename Kernel>
cudaError_t launch_fwd_common(Kernel kernel, int kind, const CUtensorMap& tq, const CUtensorMap& tk,
                              const CUtensorMap& tv, const FwdParams& p, cudaStream_t stream) {
  using C = FwdCfg<D, FP8>;
  if (p.n_items < 0) return cudaErrorInvalidValue;
  cudaError_t e = cudaMemsetAsync(p.item_counter, 0, sizeof(int), stream);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const int grid = std::min(p.n_items, sm_count_fwd());
  LaunchScope scope(kind, stream);
  kernel<<<grid, kThreads, C::SMEM_BYTES, stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_fwd_d(const Problem& pb, const void* q, const void* k, const void* v, void* o, float* lse,
                         void* workspace, cudaStream_t stream) {
  using C = FwdCfg<D>;
  alignas(64) CUtensorMap tq, tk, tv;
  if (!encode_tma_3d(&tq, q, D, pb.hq, pb.total_tokens, C::PANEL, kRows) ||
      !encode_tma_3d(&tk, k, D, pb.hkv, pb.total_tokens, C::PANEL, kKeys) ||
      !encode_tma_3d(&tv, v, D, pb.hkv, pb.total_tokens, C::PANEL, kKeys))
    return cudaErrorInvalidValue;
  const FwdParams p = fwd_params<D, false>(pb, o, lse, workspace);
  return launch_fwd_common<D, false>(fwd_bf16_sm100<D>, K_FWD_BF16, tq, tk, tv, p, stream);
}

}  // namespace

cudaError_t launch_fwd_bf16(const Problem& pb, const void* q, const void* k, const void* v, void* o, float* lse,
                            void* workspace, cudaStream_t stream) {
  if (pb.total_tokens == 0 || pb.batch == 0 || pb.max_seqlen == 0) return cudaSuccess;
  switch (pb.d) {
    case 32: return launch_fwd_d<32>(pb, q, k, v, o, lse, workspace, stream);
    case 64: return launch_fwd_d<64>(pb, q, k, v, o, lse, workspace, stream);
    case 128: return launch_fwd_d<128>(pb, q, k, v, o, lse, workspace, stream);
    default: return cudaErrorInvalidValue;
  }
}

namespace {

template <int D>
cudaError_t launch_fwd_fp8_d(const Problem& pb, const void* q8, const void* k8, const void* vt8,
                             const float* descale_q, const float* descale_k, const float* descale_v, void* o,
                             float* lse, void* workspace, cudaStream_t stream) {
  const int sp = fp8_vt_pitch(pb.cu_seqlens ? pb.max_seqlen : pb.seqlen);
  alignas(64) CUtensorMap tq, tk, tv;
  // Q8, K8: [tokens, heads, d] bytes, one d-byte swizzled row per token
  if (!encode_tma_u8_3d(&tq, q8, D, pb.hq, pb.total_tokens, (uint64_t)D, (uint64_t)pb.hq * D, D, 1, kRows) ||
      !encode_tma_u8_3d(&tk, k8, D, pb.hkv, pb.total_tokens, (uint64_t)D, (uint64_t)pb.hkv * D, D, 1, kKeys) ||
      // V^T: [batch * hkv][d][sp] bytes, boxes of 128 keys x d features
      !encode_tma_u8_3d(&tv, vt8, sp, D, pb.batch * pb.hkv, (uint64_t)sp, (uint64_t)D * sp, kKeys, D, 1))
    return cudaErrorInvalidValue;
  FwdParams p = fwd_params<D, true>(pb, o, lse, workspace);
  p.descale_q = descale_q;
  p.descale_k = descale_k;
  p.descale_v = descale_v;
  return launch_fwd_common<D, true>(fwd_fp8_sm100<D>, K_FWD_FP8, tq, tk, tv, p, stream);
}

}  // namespace

cudaError_t launch_fwd_fp8(const Problem& pb, const void* q8, const void* k8, const void* vt8,
                           const float* descale_q, const float* descale_k, const float* descale_v, void* o,
                           float* lse, void* workspace, cudaStream_t stream) {
  if (pb.total_tokens == 0 || pb.batch == 0 || pb.max_seqlen == 0) return cudaSuccess;
  switch (pb.d) {
    case 64:
      return launch_fwd_fp8_d<64>(pb, q8, k8, vt8, descale_q, descale_k, descale_v, o, lse, workspace, stream);
    case 128:
      return launch_fwd_fp8_d<128>(pb, q8, k8, vt8, descale_q, descale_k, descale_v, o, lse, workspace, stream);
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace attn
