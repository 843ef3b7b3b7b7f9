// fa_fwd_pair.cuh -- the head-dim-256 forward on CTA pairs (cta_group::2).
//
// "flashrt/fa4-cute-runtime" names a dedicated Blackwell D256 forward path on
// two CTAs.  Here two CTAs of a cluster, on two SMs, share every tensor-core
// instruction of one work unit of 256 packed query rows: CTA r holds rows
// [128 r, 128 r + 128) of the unit's Q tile and of its score and output
// accumulators, and the MMAs (M = 256) are issued by one thread of the even
// CTA for both.  The B operands are split by columns: for S = Q K^T each CTA
// holds 64 of a key tile's 128 keys (all 256 dims), for O += P V each CTA
// holds 128 of V's 256 dims (all 128 keys).  So a 128-key tile costs each SM
// 64 KB of shared memory instead of 128 KB, the score MMAs run at N = 128
// (the single-CTA kernel at D = 256 fits only 64-key tiles, whose N = 64
// score MMAs issue slower than they execute), and two key tiles stay in
// flight next to the 64 KB Q tile.
//
// Per CTA: warp 0 loads (its own Q rows and operand halves; the copies count
// their bytes on the even CTA's barriers), warp 1 issues the pair's MMAs
// (even CTA) or only follows the unit ring (odd CTA), warp 2 schedules (both
// CTAs decode the same static schedule of units, one unit per pair), warps
// 4..7 run the softmax of the CTA's 128 rows (role_softmax with trow = rank;
// its "P ready" and "O free" arrivals go to the even CTA).  Commits of the
// pair's MMAs arrive on the same barrier offset in both CTAs (multicast
// commit).  Every wait is bounded; the CTAs meet at cluster barriers after
// set-up and before the tensor memory is released.
#pragma once

#include "fa_fwd_kernel.cuh"

namespace fab {

template <bool HALF_, bool MODS_>
struct FwdPairCfg {
  static constexpr int D = 256, BN = 128, NQ = 1, NS = 2;
  static constexpr bool HALF = HALF_, PARTIAL = false, MODS = MODS_;
  static constexpr bool k2SM = true;
  static constexpr int kUnitTiles = 2;  // rows of a unit: 2 x 128, one tile per CTA
  static constexpr bool kSplitPV = false, kSplitS = false, kSepP = false;
  static constexpr int kCE = 64, kCB = 128, kChunks = D / kCE;
  static constexpr uint32_t kSBO = 8 * kCB, kLayout = 2u;  // SWIZZLE_128B
  static constexpr int kKPerChunk = kCE / 16;
  static constexpr int kQTile = kBM * D * 2;          // 64 KB
  static constexpr int kQChunk = kBM * kCB;           // 16 KB
  static constexpr int kKHalfKeys = BN / 2;           // keys of K held per CTA
  static constexpr int kKChunk = kKHalfKeys * kCB;    // 8 KB: 64 keys x 64 dims
  static constexpr int kVHalfDims = D / 2;            // dims of V held per CTA
  static constexpr int kVChunk = BN * kCB;            // 16 KB: 128 keys x 64 dims
  static constexpr int kItem = 32768;                 // one K half or one V half
  static_assert(kKChunk * kChunks == kItem && kVChunk * (kVHalfDims / kCE) == kItem, "items");
  static constexpr int kRing = 4;  // items in flight, K(n), V(n), K(n+1), ... in turn
  static constexpr int kOStride = D;
  static constexpr int kQOff = 0, kRingOff0 = kQTile;
  static constexpr int kBarOff = kRingOff0 + kRing * kItem;
  // barriers.  bQFull, bFull: on the even CTA, two arrivals (one producer per
  // CTA) plus both CTAs' bytes; bPFull, bOEmpty: on the even CTA, one arrival
  // per softmax warp of either CTA; the others are local to each CTA
  static constexpr int bQFull = 0, bQEmpty = 1, bFull = 2, bEmpty = bFull + kRing,
                       bSFull = bEmpty + kRing, bPFull = bSFull + NS, bOFull = bPFull + NS,
                       bOEmpty = bOFull + NS, bSRead = bOEmpty + 1, bPHalf = bSRead + 1,
                       bDrain = bPHalf + 1, bUFull = bDrain + 1, bUEmpty = bUFull + kUnitRing,
                       kNumBars = bUEmpty + kUnitRing;
  static constexpr uint32_t kUnitConsumers = 2 + 4;  // producer, MMA warp, 4 softmax warps
  static constexpr int kSlotOff = kBarOff + kNumBars * 8;
  static constexpr int kSchedOff = kSlotOff + 16;
  static constexpr int kSchedRoom = 232448 - 1024 - kSchedOff - 16 - 16 - kUnitRing * kUnitBytes;
  static constexpr int kMaxSchedB = (kSchedRoom / 12 - 1) > 256 ? 256 : (kSchedRoom / 12 - 1);
  static constexpr int kRingOff = (kSchedOff + 16 + 12 * (kMaxSchedB + 1) + 15) / 16 * 16;
  static constexpr int kSmemBytes = kRingOff + kUnitRing * kUnitBytes + 1024;
  static constexpr int kThreads = 256;
  static constexpr uint32_t kTmemCols = 512;
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert(NS * BN + D <= 512, "tensor memory budget");
  __host__ __device__ static constexpr int s_col(int, int b) { return b * BN; }
  __host__ __device__ static constexpr int o_col(int) { return NS * BN; }
  __host__ __device__ static constexpr int p_col(int t, int b) { return s_col(t, b); }
  // ring item i (K(n) = 2n, V(n) = 2n + 1): slot and phase parity
  __host__ __device__ static constexpr uint32_t slot(uint32_t i) { return i % kRing; }
  __host__ __device__ static constexpr uint32_t par(uint32_t i) { return (i / kRing) & 1u; }
};

// ---------------------------------------------------------------------------
// producer (both CTAs): this CTA's Q rows, K half (keys [64 r, 64 r + 64) of
// each tile) and V half (dims [128 r, 128 r + 128)); bytes counted on the
// even CTA's barriers
// ---------------------------------------------------------------------------
template <class C>
__device__ __forceinline__ void role_producer_pair(const FwdParams &p, uint32_t sb, uint32_t rank) {
  auto bar = [&](int i) { return sb + C::kBarOff + 8u * i; };
  auto bar0 = [&](int i) { return mapa_cluster(bar(i), 0); };
  uint32_t q_cnt = 0, items = 0;
  bool ok = true;
  const bool leader = (threadIdx.x & 31u) == 0;
  uint32_t ucnt = 0;
  Unit U;
  while (ok && next_unit<C>(p, sb, ucnt, U, ok, true)) {
    if (U.nb == 0) continue;
    ok = __all_sync(0xffffffffu, mbar_wait(bar(C::bQEmpty), (q_cnt & 1u) ^ 1u, p.err, p.timeout_ns));
    if (!ok) break;
    // rows of this CTA's tile (past the sequence's end they are loaded but never stored)
    const int tok = U.q_start + (U.row0 + (int)rank * kBM) / p.P;
    if (leader) {
      const uint32_t full = bar0(C::bQFull);
      mbar_arrive_expect_tx_cluster(full, C::kQTile);
#pragma unroll
      for (int c = 0; c < C::kChunks; ++c)
        tma_load_3d_pair(sb + C::kQOff + c * C::kQChunk, &p.tm_q, c * C::kCE, U.hq0, tok, full);
    }
    __syncwarp();
    ++q_cnt;
    for (int n = 0; n < U.nb && ok; ++n) {
      const int key0 = U.k_start + U.kv_lo + n * C::BN;
#pragma unroll
      for (int kv = 0; kv < 2 && ok; ++kv, ++items) {
        const uint32_t s = C::slot(items);
        ok = __all_sync(0xffffffffu, mbar_wait(bar(C::bEmpty + s), C::par(items) ^ 1u, p.err,
                                               p.timeout_ns));
        if (!ok) break;
        if (leader) {
          const uint32_t full = bar0(C::bFull + s);
          const uint32_t dst = sb + C::kRingOff0 + s * C::kItem;
          mbar_arrive_expect_tx_cluster(full, C::kItem);
          if (kv == 0) {  // K half: 4 chunks of 64 dims x 64 keys
#pragma unroll
            for (int c = 0; c < C::kChunks; ++c)
              tma_load_3d_pair(dst + c * C::kKChunk, &p.tm_k, c * C::kCE, U.hk,
                               key0 + (int)rank * C::kKHalfKeys, full);
          } else {        // V half: 2 chunks of 64 dims x 128 keys
#pragma unroll
            for (int c = 0; c < C::kVHalfDims / C::kCE; ++c)
              tma_load_3d_pair(dst + c * C::kVChunk, &p.tm_v,
                               (int)rank * C::kVHalfDims + c * C::kCE, U.hk, key0, full);
          }
        }
        __syncwarp();
      }
    }
  }
  if (!ok && rank == 0) {
    // Drain: the even CTA's full barriers count both CTAs' copies; let the
    // latest copy of every slot land before the pair leaves.
    const uint64_t drain_ns = 200000000ull;
    for (uint32_t it = (items > C::kRing ? items - C::kRing : 0); it < items; ++it)
      mbar_wait_drain(bar(C::bFull + C::slot(it)), C::par(it), drain_ns);
    if (q_cnt) mbar_wait_drain(bar(C::bQFull), (q_cnt - 1) & 1u, drain_ns);
  }
}

// ---------------------------------------------------------------------------
// MMA issuer of the pair (warp 1 of the even CTA; the elected lane issues)
// ---------------------------------------------------------------------------
template <class C>
__device__ __forceinline__ void role_mma_pair(const FwdParams &p, uint32_t sb, uint32_t tmem) {
  auto bar = [&](int i) { return sb + C::kBarOff + 8u * i; };
  // M = 256 over the pair; N = 128 keys (S) or 256 dims (O)
  constexpr uint32_t idesc_s = instr_desc<C::HALF>(2 * kBM, C::BN, false, false);
  constexpr uint32_t idesc_pv = instr_desc<C::HALF>(2 * kBM, C::D, false, true);
  uint32_t q_cnt = 0, s_cnt = 0, u_cnt = 0, items = 0;
  bool ok = true;
  auto wait_full = [&](uint32_t it) -> bool {
    return __all_sync(0xffffffffu, mbar_wait_cluster(bar(C::bFull + C::slot(it)), C::par(it), p.err,
                                                      p.timeout_ns));
  };
  // S(g) = Q K(n)^T from ring item it
  auto issue_s = [&](uint32_t g, uint32_t it) {
    const uint32_t ka = sb + C::kRingOff0 + C::slot(it) * C::kItem;
    const uint32_t d_tmem = tmem + C::s_col(0, g % C::NS);
#pragma unroll
    for (int kk = 0; kk < C::D / 16; ++kk) {
      const uint32_t off = (kk % C::kKPerChunk) * 32;
      const uint64_t a = smem_desc(sb + C::kQOff + (kk / C::kKPerChunk) * C::kQChunk + off, 16,
                                   C::kSBO, C::kLayout);
      const uint64_t b = smem_desc(ka + (kk / C::kKPerChunk) * C::kKChunk + off, 16, C::kSBO,
                                   C::kLayout);
      tc_mma_ss_pair_elect(d_tmem, a, b, idesc_s, kk > 0 ? 1u : 0u);
    }
    tc_commit_pair_both_elect(bar(C::bSFull + g % C::NS));
  };
  // O += P(g) V(n) from ring item it (P over S(g)'s columns)
  auto issue_pv = [&](uint32_t g, uint32_t it, bool first) {
    const uint32_t va = sb + C::kRingOff0 + C::slot(it) * C::kItem;
    const uint32_t p_tmem = tmem + C::p_col(0, g % C::NS);
    const uint32_t d_tmem = tmem + C::o_col(0);
#pragma unroll
    for (int kk = 0; kk < C::BN / 16; ++kk) {
      const uint64_t b = smem_desc(va + kk * 16 * C::kCB, C::kVChunk, C::kSBO, C::kLayout);
      tc_mma_ts_pair_elect(d_tmem, p_tmem + kk * 8, b, idesc_pv, (first && kk == 0) ? 0u : 1u);
    }
    tc_commit_pair_both_elect(bar(C::bOFull + g % C::NS));
  };

  uint32_t ucnt = 0;
  Unit U;
  while (ok && next_unit<C>(p, sb, ucnt, U, ok, true)) {
    if (U.nb == 0) continue;
    const int nb = U.nb;
    const uint32_t sbase = s_cnt, ib = items;  // K(n) = item ib + 2n, V(n) = ib + 2n + 1
    ok = __all_sync(0xffffffffu, mbar_wait_cluster(bar(C::bQFull), q_cnt & 1u, p.err, p.timeout_ns));
    ++q_cnt;
    if (!ok) break;
    tc_fence_after();
    ok = wait_full(ib);
    if (!ok) break;
    tc_fence_after();
    issue_s(sbase, ib);
    if (nb == 1) tc_commit_pair_both_elect(bar(C::bQEmpty));
    tc_commit_pair_both_elect(bar(C::bEmpty + C::slot(ib)));
    for (int n = 0; n < nb && ok; ++n) {
      const uint32_t g = sbase + n;
      if (n + 1 < nb) {  // S of the next key tile into the other buffer
        const uint32_t kit = ib + 2 * (n + 1);
        ok = wait_full(kit);
        if (!ok) break;
        tc_fence_after();
        issue_s(g + 1, kit);
        if (n + 1 == nb - 1) tc_commit_pair_both_elect(bar(C::bQEmpty));
        tc_commit_pair_both_elect(bar(C::bEmpty + C::slot(kit)));
      }
      const uint32_t vit = ib + 2 * n + 1;
      ok = wait_full(vit);
      if (!ok) break;
      if (n == 0) {  // both CTAs' epilogues of the previous unit have read O
        ok = __all_sync(0xffffffffu, mbar_wait_cluster(bar(C::bOEmpty), (u_cnt & 1u) ^ 1u, p.err,
                                                        p.timeout_ns));
        if (!ok) break;
      }
      ok = __all_sync(0xffffffffu, mbar_wait_cluster(bar(C::bPFull + g % C::NS), (g / C::NS) & 1u,
                                                      p.err, p.timeout_ns));
      if (!ok) break;
      tc_fence_after();
      issue_pv(g, vit, n == 0);
      tc_commit_pair_both_elect(bar(C::bEmpty + C::slot(vit)));
    }
    items += 2 * nb;
    s_cnt += nb;
    ++u_cnt;
  }
  // every MMA this thread issued completes before tensor memory is released
  tc_commit_pair_elect(bar(C::bDrain));
  mbar_wait_drain(bar(C::bDrain), 0, ok ? p.timeout_ns : 200000000ull);
}

// warp 1 of the odd CTA: follows the unit ring (one of its consumers)
template <class C>
__device__ __forceinline__ void role_follow_units(const FwdParams &p, uint32_t sb) {
  uint32_t ucnt = 0;
  bool ok = true;
  Unit U;
  while (ok && next_unit<C>(p, sb, ucnt, U, ok, true)) {
  }
}

template <class C>
__global__ void __launch_bounds__(C::kThreads, 1) fa_fwd_pair_kernel(const __grid_constant__ FwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const int warp = warp_id_sync();
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();

  if (warp == 0 && lane == 0) {
    for (int b = 0; b < C::kNumBars; ++b) {
      uint32_t cnt = 1;
      if (b == C::bQFull || (b >= C::bFull && b < C::bFull + C::kRing)) cnt = 2;
      if (b >= C::bPFull && b < C::bPFull + C::NS) cnt = 8;  // 4 warps x 2 CTAs
      if (b == C::bOEmpty) cnt = 8;
      if (b >= C::bUEmpty && b < C::bUEmpty + kUnitRing) cnt = C::kUnitConsumers;
      mbar_init(sb + C::kBarOff + 8u * b, cnt);
    }
    fence_mbar_init_cluster();
    tma_prefetch_desc(&p.tm_q);
    tma_prefetch_desc(&p.tm_k);
    tma_prefetch_desc(&p.tm_v);
  }
  if (warp == 1) {
    tmem_alloc_pair(sb + C::kSlotOff, C::kTmemCols);
    tmem_relinquish_pair();
  }
  Sched sch;
  {
    int *base = reinterpret_cast<int *>(smem + C::kSchedOff);
    sch.n_units = base;
    sch.sorted_b = base + 4;
    sch.nt = sch.sorted_b + (C::kMaxSchedB + 1);
    sch.seg_start = sch.nt + (C::kMaxSchedB + 1);
  }
  if (warp == 2 && p.compact) build_sched<C::kUnitTiles>(p, sch, lane);
  // both CTAs' barriers initialised and tensor memory allocated before any
  // arrival crosses between them
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + C::kSlotOff);

  if (warp < 4) {
    if (warp == 0) {
      role_producer_pair<C>(p, sb, rank);
    } else if (warp == 1) {
      if (rank == 0)
        role_mma_pair<C>(p, sb, tmem);
      else
        role_follow_units<C>(p, sb);
    } else if (warp == 2) {
      role_scheduler<C>(p, sch, sb);
    }
  } else {
    role_softmax<C>(p, sb, tmem, 0, static_cast<int>(rank));
  }
  __syncwarp();
  tc_fence_before();
  cluster_sync_all();  // no CTA leaves while its pair may still reach its memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, C::kTmemCols);
  }
}

}  // namespace fab
