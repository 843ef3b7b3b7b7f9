// fa_fwd_kernel.cuh -- the attention forward kernel for sm_100a.
//
// Computes O = softmax(scale * Q K^T + bias + mask) V and its log-sum-exp
// tile by tile with an online softmax, so the score matrix never leaves the
// chip.  The operation, the distance rule and the layouts follow the pages:
// "mgoin/tml-fa4" (argument contract: varlen layout, cu_seqlens, the distance
// d = i + (k_len - q_len) - j, rel_bias added for 0 <= d < rel_extent, causal
// meaning of d) and "flashrt/fa4-cute-runtime" ((out, lse) results,
// seqused_k, packed GQA heads).  The online softmax (running max, normaliser,
// P.V accumulation) is the loop that "ATFlash-Kernel-FA4" (What the window
// does) describes.
//
// Structure of one CTA (persistent; grid = number of SMs):
//
//   warp 2      tile scheduler: decodes this CTA's work units (a static snake
//               over an ordered unit list, see decode_unit / unit_of) and
//               publishes them, one record each, through a small ring in
//               shared memory that the other roles read in the same order.
//   warp 0      TMA producer: Q tiles once per unit, then K and V tiles of
//               BN keys through shared-memory rings (separate K and V rings,
//               or one ring that K and V tiles take in turn).
//   warp 1      MMA issuer (the warp's elected lane): S = Q K^T (SS form, both operands
//               K-major in swizzled shared memory) into tensor memory,
//               and O += P V (TS form: P read from tensor memory where it
//               overwrites S, V MN-major in shared memory).  Also owns the
//               tensor-memory allocation.
//   warp 3      idle.
//   warps 4..   one 128-thread softmax warpgroup per Q tile (two or three); thread r owns
//               tile row r (= TMEM lane r).  Per KV tile it loads its score
//               row from tensor memory, adds the relative bias, applies the
//               masks, updates the running max, rescales O in tensor memory
//               only when the max has grown by more than 2^8 (conditional
//               rescaling), writes P = exp2(.) back as 16-bit pairs, and
//               after the last tile normalises O and writes O and the LSE.
//
// A Q tile holds 128 packed rows: P consecutive query heads that share one
// K/V head (P = Hq/Hkv when that divides 128, else 1) at 128/P consecutive
// positions, loaded with one 3-D TMA box {64, P, 128/P} per 64 columns
// (128-byte swizzle) or, for head dims that are not a multiple of 64, one
// {16, P, 128/P} box per 16 columns (32-byte swizzle).  The kernel width D
// may exceed the tensors' head dim: the loads fill the extra columns with
// zeros and the epilogue stores only the tensors' columns.
//
// Configurations (FwdCfg<D, BN, NQ, NS, KST, VST, HALF, PARTIAL, MODS>): two
// Q tiles per CTA with one S buffer each (throughput; three, with 64-key
// tiles from width 48 up, for problems of width <= 96 without a relative
// bias), one Q tile with a
// double-buffered S (latency-bound calls, D = 256, and the split-KV partial
// kernels, which write normalised fp32 partials for the merge kernel), and,
// for each, a MODS kernel that adds the left window bound and the soft-cap.
//
// Every wait is bounded (see mbar_wait); a role that gives up records the
// timeout in the error word (FwdParams::err), drains what it has in flight,
// and leaves its loops.
#pragma once

#include <cuda_fp16.h>

#include "sm100_ptx.cuh"

namespace fab {

constexpr int kBM = 128;  // rows per Q tile = TMEM lanes

// Of every 8 pairs of columns, this many take their exponential on the FMA
// pipe (ex2_poly2) rather than the MUFU unit, which at D = 128 is otherwise
// as loaded as the tensor core (one exponential per 4*D tensor-core flops).
#ifndef FA_POLY_PAIRS
#define FA_POLY_PAIRS 1
#endif
constexpr int kPolyPairs = FA_POLY_PAIRS;

// P = 2^(s * sl2 - mc) for the N columns [OFF, OFF + N) of a row, rounded to
// 16-bit pairs into pk; returns the sum of the unrounded values.  kPoly
// sends kPolyPairs of every 8 pairs through ex2_poly2, which needs finite
// scores (no masked column).
template <bool kHalf, bool kPoly, int OFF, int N, int M>
__device__ __forceinline__ float exp_pack(const float (&s)[M], float sl2, float mc,
                                          uint32_t (&pk)[N / 2]) {
  const uint64_t sc = f2(sl2, sl2), nm = f2(-mc, -mc);
  uint64_t acc0 = f2(0.f, 0.f), acc1 = acc0;
#pragma unroll
  for (int q = 0; q < N / 2; ++q) {
    float x0, x1, y0, y1;
    f2_split(ffma2(f2(s[OFF + 2 * q], s[OFF + 2 * q + 1]), sc, nm), x0, x1);
    if (kPoly && (q % 8) < kPolyPairs) {
      ex2_poly2(x0, x1, y0, y1);
    } else {
      y0 = ex2_approx(x0);
      y1 = ex2_approx(x1);
    }
    if (q & 1)
      acc1 = fadd2(acc1, f2(y0, y1));
    else
      acc0 = fadd2(acc0, f2(y0, y1));
    pk[q] = pack2<kHalf>(y0, y1);
  }
  float a, b, c, d;
  f2_split(acc0, a, b);
  f2_split(acc1, c, d);
  return (a + b) + (c + d);
}

// Soft-cap of N scores in raw-score units: x -> a * tanh(b * x), through the
// hardware tanh (one MUFU operation per score; built from an exponential and
// a reciprocal it took two, and the local-window + soft-cap workload ran 1.6x
// slower).  Its relative error, about 2^-11, moves a capped score by at most
// cap * 2^-11 in scaled units: the parity gates hold (softcap tests).
template <int N>
__device__ __forceinline__ void softcap_all(float (&x)[N], float a, float b) {
#pragma unroll
  for (int e = 0; e < N; ++e) x[e] = a * tanh_approx(b * x[e]);
}

// Row max of the N columns [OFF, OFF + N) over four independent chains of
// three-input maxima.
template <int OFF, int N, int M>
__device__ __forceinline__ float row_max(const float (&s)[M]) {
  float m4[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) m4[k] = fmaxf(s[OFF + 2 * k], s[OFF + 2 * k + 1]);
#pragma unroll
  for (int c = 8; c < N; c += 8)
#pragma unroll
    for (int k = 0; k < 4; ++k) m4[k] = fmax3(m4[k], s[OFF + c + 2 * k], s[OFF + c + 2 * k + 1]);
  return fmax3(m4[0], m4[1], fmaxf(m4[2], m4[3]));
}
constexpr int kUnitRing = 1;      // published units in flight (one: a unit is published when every role has taken the one before)
constexpr int kUnitBytes = 64;    // one unit record in shared memory

struct FwdParams {
  CUtensorMap tm_q, tm_k, tm_v;  // 3-D maps over [tokens, heads, D]
  void *out;                     // final output (input dtype), packed [tok, Hq, D]
  float *lse;                    // final LSE, or nullptr
  float *o_part;                 // split partials [splits][tok*Hq][D] fp32
  float *lse_part;               // split partial LSE [splits][tok*Hq]
  const int *cu_q, *cu_k;        // varlen offsets, nullptr when dense
  const int *seqused_k;          // nullptr or [B]
  // nullptr or [B]: keys of the whole sequence that follow the ones this
  // call holds (a key shard); they move every row's diagonal that far right
  const int *k_after;
  const uint16_t *rel_bias;      // nullptr or [tok, Hq, R]
  int R;
  int d_out;         // head dim of the tensors (the kernel's D, or less with zero padding)
  int st32;          // 1: output rows are 32-byte aligned (32-byte stores in the epilogue)
  int B, Sq, Sk, Hq, Hkv, G, P, lgP, n_groups;
  int total_q, total_k;
  int max_q;         // longest q length the launch is sized for (max_seqlen_q, or Sq)
  int n_mblk;        // CTA tiles per (batch, head group, split)
  int num_splits;
  int split_keys;    // keys per split (multiple of BN); >= any k_len when 1 split
  int causal;
  // window by distance d = i + delta - j from the row's diagonal: a key is
  // masked when d > wl (wl >= 0) or -d > wr (wr >= 0; causal makes wr 0)
  int wl, wr;
  // soft-cap in raw-score units: s -> cap_a * tanh(cap_b * s) when cap_a > 0
  float cap_a, cap_b;
  int m_major;       // unit order: 1 = largest tile index first over all heads
  int compact;       // 1: causal units enumerated without empty ones (see Sched)
  int lse_dense;     // 1: lse [B, Hq, Sq]; 0: lse [Hq, total_q]
  int num_units;
  float scale_log2;  // softmax_scale * log2(e)
  float inv_scale;   // 1 / softmax_scale (bias is folded into raw-score units)
  float thr_raw;     // rescale threshold 8 (log2 units) in raw-score units
  unsigned long long timeout_ns;
  // the library's device error word (timeouts, broken input contracts);
  // fa_check_device_error reads and clears it
  unsigned *err;
};

// One work unit: NQ Q tiles of one (batch, head group) and one key split.
struct Unit {
  int b, hq0, hk, split;
  int q_start, q_len, k_start, k_len, delta;
  int row0;          // first packed row of tile 0 within the sequence
  int kv_lo, kv_hi;  // key range handled by this unit
  int nb;            // KV tiles
  unsigned active;   // bit t: tile t holds at least one valid row
};

// Compact heaviest-first schedule of causal units, built per CTA in shared
// memory.  Sequences are ranked by their number of tile levels nt (a level is
// one 256-row tile index m, over all head groups and splits); with nt sorted
// in decreasing order, levels m in [nt[j+1], nt[j]) exist for exactly the
// sequences of rank 0..j.  Segment j lists those levels from the top down, so
// the whole list runs from the heaviest (largest m) unit to the lightest and
// holds no unit without rows.
struct Sched {
  int *n_units;    // [1]
  int *sorted_b;   // [B]      batch index by rank
  int *nt;         // [B + 1]  levels of the sequence of each rank, nt[B] = 0
  int *seg_start;  // [B + 1]  first unit of each segment
};

__device__ __forceinline__ int seq_tiles(const FwdParams &p, int b, int rows_per_unit) {
  const int ql = p.cu_q != nullptr ? __ldg(p.cu_q + b + 1) - __ldg(p.cu_q + b) : p.Sq;
  return ql <= 0 ? 0 : (int)(((long long)ql * p.P + rows_per_unit - 1) / rows_per_unit);
}

// Extents of sequence b: its first query token and length, its first key
// token and the number of keys it uses.  Checks the input contract of
// "mgoin/tml-fa4", argument contract (cu_seqlens [B+1], nondecreasing from
// 0, last entry the total; max_seqlen_q the largest q length) and the bound
// of seqused_k (at most the sequence's keys).  A sequence that breaks it gets
// kErrInput recorded and `false`: its units are skipped, so nothing of it is
// read or written out of range.
__device__ __forceinline__ bool seq_extents(const FwdParams &p, int b, int &q_start, int &q_len,
                                            int &k_start, int &k_len) {
  bool ok = true;
  if (p.cu_q != nullptr) {
    const int q0 = __ldg(p.cu_q + b), q1 = __ldg(p.cu_q + b + 1);
    const int k0 = __ldg(p.cu_k + b), k1 = __ldg(p.cu_k + b + 1);
    ok = q0 >= 0 && q1 >= q0 && q1 <= p.total_q && k0 >= 0 && k1 >= k0 && k1 <= p.total_k &&
         q1 - q0 <= p.max_q && (b != p.B - 1 || (q1 == p.total_q && k1 == p.total_k));
    q_start = q0;
    q_len = q1 - q0;
    k_start = k0;
    k_len = k1 - k0;
  } else {
    q_start = b * p.Sq;
    q_len = p.Sq;
    k_start = b * p.Sk;
    k_len = p.Sk;
  }
  if (p.seqused_k != nullptr) {
    const int su = __ldg(p.seqused_k + b);
    ok = ok && su >= 0 && su <= k_len;
    k_len = su;
  }
  if (!ok) atomicOr(p.err, kErrInput);
  return ok;
}

// Built by one warp before the CTA's first barrier.
template <int NQ>
__device__ __forceinline__ void build_sched(const FwdParams &p, const Sched &sch, int lane) {
  const int B = p.B;
  for (int b = lane; b < B; b += 32) {
    int qs, ql, ks, kl;
    (void)seq_extents(p, b, qs, ql, ks, kl);  // records a broken contract (units are skipped later)
    const int nb = seq_tiles(p, b, NQ * kBM);
    int rank = 0;
    for (int o = 0; o < B; ++o) {
      const int no = seq_tiles(p, o, NQ * kBM);
      rank += (no > nb) || (no == nb && o < b);
    }
    sch.sorted_b[rank] = b;
    sch.nt[rank] = nb;
  }
  __syncwarp();
  if (lane == 0) {
    sch.nt[B] = 0;
    const int W = p.n_groups * p.num_splits;
    int start = 0;
    for (int j = 0; j < B; ++j) {
      sch.seg_start[j] = start;
      start += (sch.nt[j] - sch.nt[j + 1]) * (j + 1) * W;
    }
    sch.seg_start[B] = start;
    *sch.n_units = start;
  }
}

// Unit u -> (batch, head group, tile index, split).  Causal problems are
// enumerated tile-index-major from the last (heaviest) tile down, so that the
// units come roughly sorted by decreasing work across all sequences and
// heads; other problems keep all tiles of one (batch, head group) together so
// that concurrently running CTAs share that head's K/V in L2.
template <int NQ, int BN>
__device__ __forceinline__ bool decode_unit(const FwdParams &p, const Sched &sch, int u, Unit &U) {
  int mblk, grp;
  if (p.compact) {
    int lo = 0, hi = p.B - 1;  // last segment starting at or before u
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (sch.seg_start[mid] <= u) lo = mid; else hi = mid - 1;
    }
    const int j = lo;
    const int W = p.n_groups * p.num_splits;
    const int per_level = (j + 1) * W;
    const int local = u - sch.seg_start[j];
    const int lvl = local / per_level;
    mblk = sch.nt[j] - 1 - lvl;
    int rem = local - lvl * per_level;
    const int bi = rem / W;
    U.b = sch.sorted_b[bi];
    rem -= bi * W;
    U.split = rem % p.num_splits;
    grp = rem / p.num_splits;
  } else if (p.m_major) {
    const int per_m = p.B * p.n_groups * p.num_splits;
    const int m_rev = u / per_m;
    int rest = u - m_rev * per_m;
    U.split = rest % p.num_splits;
    rest /= p.num_splits;
    grp = rest % p.n_groups;
    U.b = rest / p.n_groups;
    mblk = p.n_mblk - 1 - m_rev;
  } else {
    mblk = u % p.n_mblk;
    int rest = u / p.n_mblk;
    U.split = rest % p.num_splits;
    rest /= p.num_splits;
    grp = rest % p.n_groups;
    U.b = rest / p.n_groups;
  }
  U.hq0 = grp * p.P;
  U.hk = U.hq0 / p.G;
  if (!seq_extents(p, U.b, U.q_start, U.q_len, U.k_start, U.k_len)) return false;
  U.row0 = mblk * NQ * kBM;
  if (U.row0 / p.P >= U.q_len) return false;  // no row of this unit exists
  U.active = 0;
#pragma unroll
  for (int t = 0; t < NQ; ++t)
    if ((U.row0 + t * kBM) / p.P < U.q_len) U.active |= 1u << t;
  U.delta = U.k_len - U.q_len;
  if (p.k_after != nullptr) U.delta += min(max(__ldg(p.k_after + U.b), 0), 1 << 30);
  long long lo = (long long)U.split * p.split_keys;
  long long hi = min((long long)U.k_len, lo + p.split_keys);
  // keys no row of the unit admits are not visited: the window (causal is
  // wr = 0) bounds them on both sides
  if (p.wr >= 0) {
    const int i_max = min(U.q_len - 1, (U.row0 + NQ * kBM - 1) / p.P);
    hi = min(hi, (long long)i_max + U.delta + p.wr + 1);
  }
  if (p.wl >= 0) {
    const int i_min = U.row0 / p.P;
    lo = max(lo, (long long)i_min + U.delta - p.wl);
  }
  U.kv_lo = (int)lo;
  U.kv_hi = (int)max(hi, lo);
  U.nb = (U.kv_hi - U.kv_lo + BN - 1) / BN;
  return true;
}

// The k-th unit of this CTA in a static schedule of whole rounds of gridDim.x
// units whose direction alternates (a "snake"): with units sorted by
// decreasing work, each CTA's heavy and light picks even out.
__device__ __forceinline__ int unit_of(int k, int pair_shift = 0) {
  // CTA pairs (pair_shift 1) walk the schedule together, one unit per pair
  const int G = static_cast<int>(gridDim.x) >> pair_shift;
  const int c = static_cast<int>(blockIdx.x) >> pair_shift;
  return k * G + ((k & 1) ? (G - 1 - c) : c);
}

// Shared-memory matrix descriptor (sm_100 layout: start address, leading and
// stride byte offsets in 16-byte units, version 1, layout type in the top
// bits: 2 = SWIZZLE_128B, 6 = SWIZZLE_32B).
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo,
                                              uint32_t layout) {
  uint64_t d = 0;
  d |= (uint64_t)((addr & 0x3FFFFu) >> 4);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;
  d |= (uint64_t)(layout & 7u) << 61;
  return d;
}

// Instruction descriptor of tcgen05.mma kind::f16 with an fp32 accumulator.
template <bool kHalf>
__host__ __device__ constexpr uint32_t instr_desc(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4)                                  // D format: f32
         | ((kHalf ? 0u : 1u) << 7)                 // A: f16 / bf16
         | ((kHalf ? 0u : 1u) << 10)                // B: f16 / bf16
         | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16)
         | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

template <int D_, int BN_, int NQ_, int NS_, int KST_, int VST_, bool HALF_, bool PARTIAL_,
          bool MODS_ = false>
struct FwdCfg {
  static constexpr int D = D_, BN = BN_, NQ = NQ_, NS = NS_, KST = KST_, VST = VST_;
  static constexpr bool HALF = HALF_, PARTIAL = PARTIAL_;
  // one CTA per unit (the paired-SM configuration is FwdPairCfg); a unit
  // holds NQ Q tiles
  static constexpr bool k2SM = false;
  static constexpr int kUnitTiles = NQ_;
  // score/mask modifiers beyond causal (left window bound, soft-cap): a
  // separate kernel, so that the plain one carries none of their cost
  static constexpr bool MODS = MODS_;
  // Row chunks: 64 columns with a 128-byte swizzle when D is a multiple of
  // 64; otherwise (narrow head dims, D a multiple of 16 holding a head dim
  // padded up by zero-filled loads) 16 columns with a 32-byte swizzle.
  static constexpr bool kNarrow = D % 64 != 0;
  static constexpr int kCE = kNarrow ? 16 : 64;           // columns of a chunk
  static constexpr int kCB = 2 * kCE;                     // bytes of a chunk row
  static constexpr int kChunks = D / kCE;
  static constexpr int kQTile = kBM * D * 2;      // bytes
  static constexpr int kKVTile = BN * D * 2;
  static constexpr int kQChunk = kBM * kCB;       // bytes of one chunk
  static constexpr int kKVChunk = BN * kCB;
  static constexpr uint32_t kSBO = 8 * kCB;       // stride of 8-row groups
  static constexpr uint32_t kLayout = kNarrow ? 6u : 2u;
  static constexpr int kKPerChunk = kCE / 16;     // 16-column MMA steps per chunk
  static constexpr int kOStride = (D + 31) / 32 * 32;  // tensor-memory columns of one O
  static constexpr int kQOff = 0;
  // K/V stages: separate rings of KST and VST slots, or (VST == 0) one ring of
  // KST slots that the K and V tiles take in turn -- K(n), V(n), K(n+1), ...
  // -- so that K(n+1) reuses the slot of V(n-1) and V(n+1) that of K(n).
  static constexpr bool kKVRing = VST == 0;
  static constexpr int kKOff = kQOff + NQ * kQTile;
  static constexpr int kVOff = kKVRing ? kKOff : kKOff + KST * kKVTile;
  static constexpr int kBarOff = kKOff + (KST + VST) * kKVTile;
  // Split P.V (single S buffer, 128-key tiles): P.V starts on the first 64
  // keys once the softmax has stored their half of P, overlapping the second
  // half's exponentials; the rest follows the whole of P.
  static constexpr bool kSplitPV = NS == 1 && BN == 128;
  // Split score MMA as well: P(n) fills columns [0, 64) of its tile's S
  // buffer, so the keys 64..127 of S(n+1), which land in columns [64, 128),
  // can be computed as soon as the softmax has read S(n).  Measured slower:
  // 128x64 MMAs issue at ~50 cycles for 32 of work.
  static constexpr bool kSplitS = false;
  // Separate P buffer (64 tensor-memory columns per Q tile, where S, O and P
  // fit: D <= 64): P(n) no longer overwrites S(n), so S(n+1) is computed as
  // soon as the softmax has read S(n), while it works on tile n, instead of
  // after P(n).V.  The softmax then waits for P(n-1).V before it stores P(n)
  // or rescales O.  Measured 9-15% slower at D = 16 and 64: the two tiles'
  // softmaxes then run at the same time on the same SMSPs instead of taking
  // turns, and their exponential and FMA work per SMSP does not shrink.
#ifndef FA_SEPARATE_P
#define FA_SEPARATE_P 0
#endif
  static constexpr bool kSepPWanted = FA_SEPARATE_P != 0;
  static constexpr bool kSepP = kSepPWanted && kSplitPV && NQ == 2 && !kSplitS &&
                                NQ * NS * BN + NQ * ((D + 31) / 32 * 32) + NQ * (BN / 2) <= 512;
  // barrier indices
  static constexpr int bQFull = 0, bQEmpty = NQ, bKFull = 2 * NQ, bKEmpty = bKFull + KST,
                       bVFull0 = bKEmpty + KST, bVEmpty0 = bVFull0 + VST, bSFull = bVEmpty0 + VST,
                       bVFull = kKVRing ? bKFull : bVFull0, bVEmpty = kKVRing ? bKEmpty : bVEmpty0,
                       bPFull = bSFull + NQ * NS, bOFull = bPFull + NQ * NS,
                       bOEmpty = bOFull + NQ * NS, bSRead = bOEmpty + NQ, bPHalf = bSRead + NQ,
                       bDrain = bPHalf + NQ,
                       bUFull = bDrain + 1, bUEmpty = bUFull + kUnitRing,
                       kNumBars = bUEmpty + kUnitRing;
  // consumers of each published unit: producer, MMA issuer, every softmax warp
  static constexpr uint32_t kUnitConsumers = 2 + 4 * NQ;
  static constexpr int kSlotOff = kBarOff + kNumBars * 8;
  // compact causal schedule: 3 int arrays of up to kMaxSchedB + 1 entries
  static constexpr int kSchedOff = kSlotOff + 16;
  static constexpr int kSchedRoom = 232448 - 1024 - kSchedOff - 16 - 16 - kUnitRing * kUnitBytes;
  static constexpr int kMaxSchedB = (kSchedRoom / 12 - 1) > 256 ? 256 : (kSchedRoom / 12 - 1);
  static constexpr int kRingOff = (kSchedOff + 16 + 12 * (kMaxSchedB + 1) + 15) / 16 * 16;
  static constexpr int kSmemBytes = kRingOff + kUnitRing * kUnitBytes + 1024;  // + alignment slack
  static constexpr int kThreads = 128 * (1 + NQ);
  // registers: with two softmax warpgroups the launch budget (65536 / 384
  // threads = 168 each) is re-split so that the softmax warps hold a whole
  // score row, or half a row plus its bias window, without spilling; the
  // modifier kernels (window bounds, soft-cap) take 224 of them.  With three
  // (65536 / 512 = 128 each) the softmax warps get 152 and work on half rows.
  static constexpr bool kSplitRegs = NQ >= 2;
  static constexpr uint32_t kRegsCtl = NQ == 3 ? 56 : (MODS_ ? 56 : 72),
                            kRegsSoftmax = NQ == 3 ? 152 : (MODS_ ? 224 : 216);
  static_assert(!kSplitRegs || 128 * kRegsCtl + 128 * NQ * kRegsSoftmax <=
                                   kThreads * ((65536 / kThreads) & ~7),
                "register split");
  static constexpr uint32_t kTmemCols = 512;
  static constexpr int kOColBase = NQ * NS * BN;
  static constexpr int kPColBase = kOColBase + NQ * kOStride;
  static_assert(kPColBase + (kSepP ? NQ * BN / 2 : 0) <= 512, "tensor memory budget");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert((D % 64 == 0 || (D % 16 == 0 && D < 128)) && BN % 32 == 0 &&
                    (BN == 64 || BN == 128), "tile shape");
  // slot and phase parity of the K tile k / V tile v (counted over the CTA's
  // whole sequence of KV tiles), and the barriers of V slots
  __host__ __device__ static constexpr uint32_t k_slot(uint32_t k) {
    return kKVRing ? (2u * k) % KST : k % KST;
  }
  __host__ __device__ static constexpr uint32_t k_par(uint32_t k) {
    return kKVRing ? ((2u * k) / KST) & 1u : (k / KST) & 1u;
  }
  __host__ __device__ static constexpr uint32_t v_slot(uint32_t v) {
    return kKVRing ? (2u * v + 1u) % KST : v % VST;
  }
  __host__ __device__ static constexpr uint32_t v_par(uint32_t v) {
    return kKVRing ? ((2u * v + 1u) / KST) & 1u : (v / VST) & 1u;
  }
  __host__ __device__ static constexpr int s_col(int t, int b) { return (t * NS + b) * BN; }
  __host__ __device__ static constexpr int o_col(int t) { return kOColBase + t * kOStride; }
  // columns of P_t(g): its own buffer, or the first half of S_t(g)'s
  __host__ __device__ static constexpr int p_col(int t, int b) {
    return kSepP ? kPColBase + t * (BN / 2) : s_col(t, b);
  }
};

// ---------------------------------------------------------------------------
// unit ring: the scheduler warp decodes each unit once and publishes it;
// producer, MMA issuer and softmax warps read the same sequence
// ---------------------------------------------------------------------------
__device__ __forceinline__ void unit_store(uint32_t addr, const Unit &U) {
  sts_v4(addr, make_uint4(U.b, U.hq0, U.hk, U.split));
  sts_v4(addr + 16, make_uint4(U.q_start, U.q_len, U.k_start, U.k_len));
  sts_v4(addr + 32, make_uint4(U.delta, U.row0, U.kv_lo, U.kv_hi));
  sts_v4(addr + 48, make_uint4(U.nb, U.active, 0u, 0u));
}

__device__ __forceinline__ void unit_load(uint32_t addr, Unit &U) {
  uint4 a = lds_v4(addr), b = lds_v4(addr + 16), c = lds_v4(addr + 32), d = lds_v4(addr + 48);
  U.b = a.x; U.hq0 = a.y; U.hk = a.z; U.split = a.w;
  U.q_start = b.x; U.q_len = b.y; U.k_start = b.z; U.k_len = b.w;
  U.delta = c.x; U.row0 = c.y; U.kv_lo = c.z; U.kv_hi = c.w;
  U.nb = (int)d.x; U.active = d.y;
}

// Next unit for one consumer.  `warp_wide`: all 32 lanes read and one
// arrival per warp is made; otherwise the calling thread alone.  Returns
// false at the end of the schedule (a record with nb < 0) or on a timeout
// (then *ok is false).
template <class C>
__device__ __forceinline__ bool next_unit(const FwdParams &p, uint32_t sb, uint32_t &cnt, Unit &U,
                                          bool &ok, bool warp_wide) {
  const uint32_t slot = cnt % kUnitRing;
  const uint32_t full = sb + C::kBarOff + 8u * (C::bUFull + slot);
  bool w = mbar_wait(full, (cnt / kUnitRing) & 1u, p.err, p.timeout_ns);
  if (warp_wide) w = __all_sync(0xffffffffu, w);
  if (!w) {
    ok = false;
    return false;
  }
  unit_load(sb + C::kRingOff + slot * kUnitBytes, U);
  if (warp_wide) __syncwarp();
  if (!warp_wide || (threadIdx.x & 31u) == 0)
    mbar_arrive(sb + C::kBarOff + 8u * (C::bUEmpty + slot));
  ++cnt;
  return U.nb >= 0;
}

template <class C>
__device__ __forceinline__ void role_scheduler(const FwdParams &p, const Sched &sch, uint32_t sb) {
  uint32_t cnt = 0;
  auto publish = [&](const Unit &U) -> bool {
    const uint32_t slot = cnt % kUnitRing;
    if (!__all_sync(0xffffffffu, mbar_wait_sleepy(sb + C::kBarOff + 8u * (C::bUEmpty + slot),
                                                  ((cnt / kUnitRing) & 1u) ^ 1u, p.err,
                                                  p.timeout_ns)))
      return false;
    if ((threadIdx.x & 31u) == 0) {  // the warp stays converged; lane 0 publishes
      unit_store(sb + C::kRingOff + slot * kUnitBytes, U);
      mbar_arrive(sb + C::kBarOff + 8u * (C::bUFull + slot));
    }
    __syncwarp();
    ++cnt;
    return true;
  };
  const int n_units = p.compact ? *sch.n_units : p.num_units;
  bool ok = true;
  constexpr int kPS = C::k2SM ? 1 : 0;
  for (int k = 0; k * ((int)gridDim.x >> kPS) < n_units && ok; ++k) {
    const int u = unit_of(k, kPS);
    Unit U;
    if (u >= n_units || !decode_unit<C::kUnitTiles, C::BN>(p, sch, u, U)) continue;
    ok = publish(U);
  }
  if (ok) {
    Unit end;
    end.b = end.hq0 = end.hk = end.split = 0;
    end.q_start = end.q_len = end.k_start = end.k_len = end.delta = end.row0 = 0;
    end.kv_lo = end.kv_hi = 0;
    end.nb = -1;
    end.active = 0u;
    publish(end);
  }
}

// ---------------------------------------------------------------------------
// producer
// ---------------------------------------------------------------------------
template <class C>
__device__ __forceinline__ void role_producer(const FwdParams &p, uint32_t sb) {
  auto bar = [&](int i) { return sb + C::kBarOff + 8u * i; };
  uint32_t q_cnt[C::NQ];
#pragma unroll
  for (int t = 0; t < C::NQ; ++t) q_cnt[t] = 0;
  uint32_t k_cnt = 0, v_cnt = 0;
  bool ok = true;
  const bool leader = (threadIdx.x & 31u) == 0;  // issues the copies; the warp stays converged
  uint32_t ucnt = 0;
  Unit U;
  while (ok && next_unit<C>(p, sb, ucnt, U, ok, true)) {
    if (U.nb == 0) continue;
#pragma unroll
    for (int t = 0; t < C::NQ; ++t) {
      if (!(U.active >> t & 1u)) continue;
      ok = __all_sync(0xffffffffu, mbar_wait(bar(C::bQEmpty + t), (q_cnt[t] & 1u) ^ 1u, p.err, p.timeout_ns));
      if (!ok) break;
      const int tok = U.q_start + (U.row0 + t * kBM) / p.P;
      if (leader) {
        mbar_arrive_expect_tx(bar(C::bQFull + t), C::kQTile);
#pragma unroll
        for (int c = 0; c < C::kChunks; ++c)
          tma_load_3d(sb + C::kQOff + t * C::kQTile + c * C::kQChunk, &p.tm_q, c * C::kCE, U.hq0, tok,
                      bar(C::bQFull + t));
      }
      __syncwarp();
      ++q_cnt[t];
    }
    for (int n = 0; n < U.nb && ok; ++n) {
      const int tok = U.k_start + U.kv_lo + n * C::BN;
      {
        const uint32_t s = C::k_slot(k_cnt);
        ok = __all_sync(0xffffffffu, mbar_wait(bar(C::bKEmpty + s), C::k_par(k_cnt) ^ 1u, p.err,
                       p.timeout_ns));
        if (!ok) break;
        if (leader) {
          mbar_arrive_expect_tx(bar(C::bKFull + s), C::kKVTile);
#pragma unroll
          for (int c = 0; c < C::kChunks; ++c)
            tma_load_3d(sb + C::kKOff + s * C::kKVTile + c * C::kKVChunk, &p.tm_k, c * C::kCE, U.hk,
                        tok, bar(C::bKFull + s));
        }
        __syncwarp();
        ++k_cnt;
      }
      {
        const uint32_t s = C::v_slot(v_cnt);
        ok = __all_sync(0xffffffffu, mbar_wait(bar(C::bVEmpty + s), C::v_par(v_cnt) ^ 1u, p.err,
                       p.timeout_ns));
        if (!ok) break;
        if (leader) {
          mbar_arrive_expect_tx(bar(C::bVFull + s), C::kKVTile);
#pragma unroll
          for (int c = 0; c < C::kChunks; ++c)
            tma_load_3d(sb + C::kVOff + s * C::kKVTile + c * C::kKVChunk, &p.tm_v, c * C::kCE, U.hk,
                        tok, bar(C::bVFull + s));
        }
        __syncwarp();
        ++v_cnt;
      }
    }
  }
  if (!ok) {
    // Drain: let every copy this warp issued land before the CTA leaves.
    const uint64_t drain_ns = 200000000ull;
    // the latest load of every slot
    if constexpr (C::kKVRing) {
      const uint32_t n_items = k_cnt + v_cnt;  // K and V tiles issued, in ring order
      for (uint32_t it = (n_items > C::KST ? n_items - C::KST : 0); it < n_items; ++it)
        mbar_wait_drain(bar(C::bKFull + it % C::KST), (it / C::KST) & 1u, drain_ns);
    } else {
      for (uint32_t i = (k_cnt > C::KST ? k_cnt - C::KST : 0); i < k_cnt; ++i)
        mbar_wait_drain(bar(C::bKFull + C::k_slot(i)), C::k_par(i), drain_ns);
      for (uint32_t i = (v_cnt > C::VST ? v_cnt - C::VST : 0); i < v_cnt; ++i)
        mbar_wait_drain(bar(C::bVFull + C::v_slot(i)), C::v_par(i), drain_ns);
    }
#pragma unroll
    for (int t = 0; t < C::NQ; ++t)
      if (q_cnt[t]) mbar_wait_drain(bar(C::bQFull + t), (q_cnt[t] - 1) & 1u, drain_ns);
  }
}

// ---------------------------------------------------------------------------
// MMA issuer (one converged warp; the elected lane issues)
// ---------------------------------------------------------------------------
template <class C>
__device__ __forceinline__ void role_mma(const FwdParams &p, uint32_t sb, uint32_t tmem) {
  auto bar = [&](int i) { return sb + C::kBarOff + 8u * i; };
  constexpr uint32_t idesc_s = instr_desc<C::HALF>(kBM, C::BN, false, false);
  constexpr uint32_t idesc_pv = instr_desc<C::HALF>(kBM, C::D, false, true);
  uint32_t q_cnt[C::NQ], s_cnt[C::NQ], u_cnt[C::NQ];
#pragma unroll
  for (int t = 0; t < C::NQ; ++t) q_cnt[t] = s_cnt[t] = u_cnt[t] = 0;
  uint32_t k_cnt = 0, v_cnt = 0;
  bool ok = true;

  // S_t(n) = Q_t K_n^T into the S buffer of global index g
  auto issue_s = [&](int t, uint32_t g, uint32_t kstage) {
    const uint32_t qa = sb + C::kQOff + t * C::kQTile;
    const uint32_t ka = sb + C::kKOff + kstage * C::kKVTile;
    const uint32_t d_tmem = tmem + C::s_col(t, g % C::NS);
#pragma unroll
    for (int kk = 0; kk < C::D / 16; ++kk) {
      // 16 elements = 32 bytes inside the swizzle atom
      const uint32_t off = (kk % C::kKPerChunk) * 32;
      const uint64_t a = smem_desc(qa + (kk / C::kKPerChunk) * C::kQChunk + off, 16, C::kSBO,
                                   C::kLayout);
      const uint64_t b = smem_desc(ka + (kk / C::kKPerChunk) * C::kKVChunk + off, 16, C::kSBO,
                                   C::kLayout);
      tc_mma_ss_elect(d_tmem, a, b, idesc_s, kk > 0 ? 1u : 0u);
    }
    tc_commit_elect(bar(C::bSFull + t * C::NS + g % C::NS));
  };
  // O_t += P_t(g) V (P in the S buffer of g, as 16-bit pairs)
  // O_t += P_t(g) V (P in the S buffer of g, as 16-bit pairs)
  auto issue_pv = [&](int t, uint32_t g, uint32_t vstage, bool first) {
    const uint32_t va = sb + C::kVOff + vstage * C::kKVTile;
    const uint32_t p_tmem = tmem + C::p_col(t, g % C::NS);
    const uint32_t d_tmem = tmem + C::o_col(t);
#pragma unroll
    for (int kk = 0; kk < C::BN / 16; ++kk) {
      // 16 keys = two 8-row groups (SBO apart); column chunks LBO apart
      const uint64_t b = smem_desc(va + kk * 16 * C::kCB, C::kKVChunk, C::kSBO, C::kLayout);
      tc_mma_ts_elect(d_tmem, p_tmem + kk * 8, b, idesc_pv, (first && kk == 0) ? 0u : 1u);
    }
    tc_commit_elect(bar(C::bOFull + t * C::NS + g % C::NS));
  };

  // split form: keys [64 hi, 64 hi + 64) of S_t into columns [64 hi, 64 hi + 64)
  constexpr uint32_t idesc_s64 = instr_desc<C::HALF>(kBM, 64, false, false);
  auto issue_s_half = [&](int t, uint32_t g, uint32_t kstage, int hi) {
    const uint32_t qa = sb + C::kQOff + t * C::kQTile;
    const uint32_t ka = sb + C::kKOff + kstage * C::kKVTile + hi * 64 * C::kCB;
    const uint32_t d_tmem = tmem + C::s_col(t, g % C::NS) + hi * 64;
#pragma unroll
    for (int kk = 0; kk < C::D / 16; ++kk) {
      const uint32_t off = (kk % C::kKPerChunk) * 32;
      const uint64_t a = smem_desc(qa + (kk / C::kKPerChunk) * C::kQChunk + off, 16, C::kSBO,
                                   C::kLayout);
      const uint64_t b = smem_desc(ka + (kk / C::kKPerChunk) * C::kKVChunk + off, 16, C::kSBO,
                                   C::kLayout);
      tc_mma_ss_elect(d_tmem, a, b, idesc_s64, kk > 0 ? 1u : 0u);
    }
  };
  // split form: O_t += P_t[:, 64 hi .. 64 hi + 64) V[64 hi .. 64 hi + 64, :]
  auto issue_pv_half = [&](int t, uint32_t g, uint32_t vstage, bool first, int hi) {
    const uint32_t va = sb + C::kVOff + vstage * C::kKVTile;
    const uint32_t p_tmem = tmem + C::p_col(t, g % C::NS);
    const uint32_t d_tmem = tmem + C::o_col(t);
#pragma unroll
    for (int k4 = 0; k4 < 4; ++k4) {
      const int kk = 4 * hi + k4;
      const uint64_t b = smem_desc(va + kk * 16 * C::kCB, C::kKVChunk, C::kSBO, C::kLayout);
      tc_mma_ts_elect(d_tmem, p_tmem + kk * 8, b, idesc_pv, (first && kk == 0) ? 0u : 1u);
    }
  };

  uint32_t ucnt = 0;
  Unit U;
  while (ok && next_unit<C>(p, sb, ucnt, U, ok, true)) {
    if (U.nb == 0) continue;
    const int nb = U.nb;
    // the last tile with rows
    const int last_t = C::NQ == 3 ? 31 - __clz(U.active) : ((U.active >> 1 & 1u) && C::NQ > 1 ? 1 : 0);
    uint32_t sbase[C::NQ];
#pragma unroll
    for (int t = 0; t < C::NQ; ++t) {
      sbase[t] = s_cnt[t];
      if (!(U.active >> t & 1u)) continue;
      ok = ok && __all_sync(0xffffffffu, mbar_wait(bar(C::bQFull + t), q_cnt[t] & 1u, p.err, p.timeout_ns));
      ++q_cnt[t];
    }
    if (!ok) break;
    tc_fence_after();
    const uint32_t kb = k_cnt, vb = v_cnt;

    // prologue: S(0) for every active tile
    ok = __all_sync(0xffffffffu, mbar_wait(bar(C::bKFull + C::k_slot(kb)), C::k_par(kb), p.err, p.timeout_ns));
    if (!ok) break;
    tc_fence_after();
#pragma unroll
    for (int t = 0; t < C::NQ; ++t) {
      if (!(U.active >> t & 1u)) continue;
      issue_s(t, sbase[t], C::k_slot(kb));
      if (nb == 1) tc_commit_elect(bar(C::bQEmpty + t));
    }
    tc_commit_elect(bar(C::bKEmpty + C::k_slot(kb)));

    for (int n = 0; n < nb && ok; ++n) {
      const uint32_t kn = kb + n + 1;  // K tile of block n+1
      if (C::NS == 2 && n + 1 < nb) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar(C::bKFull + C::k_slot(kn)), C::k_par(kn), p.err,
                       p.timeout_ns));
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int t = 0; t < C::NQ; ++t) {
          if (!(U.active >> t & 1u)) continue;
          issue_s(t, sbase[t] + n + 1, C::k_slot(kn));
          if (n + 1 == nb - 1) tc_commit_elect(bar(C::bQEmpty + t));
        }
        tc_commit_elect(bar(C::bKEmpty + C::k_slot(kn)));
      }
      const uint32_t vn = vb + n;
      bool k_next_ready = false;  // K tile n+1 waited for (split form)
      if constexpr (C::kSepP) {
        // S_t(n+1) for every tile as soon as its softmax has read S_t(n)
        if (n + 1 < nb) {
          ok = __all_sync(0xffffffffu, mbar_wait(bar(C::bKFull + C::k_slot(kn)), C::k_par(kn),
                                                 p.err, p.timeout_ns));
          if (!ok) break;
          k_next_ready = true;
#pragma unroll
          for (int t = 0; t < C::NQ; ++t) {
            if (!(U.active >> t & 1u)) continue;
            const uint32_t g = sbase[t] + n;
            ok = __all_sync(0xffffffffu, mbar_wait(bar(C::bSRead + t), g & 1u, p.err,
                                                   p.timeout_ns));
            if (!ok) break;
            tc_fence_after();
            issue_s(t, g + 1, C::k_slot(kn));  // commits the S barrier itself
            if (n + 1 == nb - 1) tc_commit_elect(bar(C::bQEmpty + t));
          }
          if (!ok) break;
          tc_commit_elect(bar(C::bKEmpty + C::k_slot(kn)));
        }
      }
      ok = __all_sync(0xffffffffu, mbar_wait(bar(C::bVFull + C::v_slot(vn)), C::v_par(vn), p.err,
                     p.timeout_ns));
      if (!ok) break;
#pragma unroll
      for (int t = 0; t < C::NQ; ++t) {
        if (!(U.active >> t & 1u)) continue;
        const uint32_t g = sbase[t] + n;
        if (n == 0) {
          ok = __all_sync(0xffffffffu, mbar_wait(bar(C::bOEmpty + t), (u_cnt[t] & 1u) ^ 1u, p.err, p.timeout_ns));
          if (!ok) break;
        }
        if constexpr (C::kSplitPV) {
          // keys 64..127 of S_t(n+1) as soon as S_t(n) has been read (split S); P.V on
          // the first 64 keys once their half of P is stored, then the rest;
          // keys 0..63 of S_t(n+1) after P.V has read P_t(n)
          const bool more = n + 1 < nb;
          if (C::kSplitS && more) {
            if (!k_next_ready) {
              ok = __all_sync(0xffffffffu, mbar_wait(bar(C::bKFull + C::k_slot(kn)),
                                                     C::k_par(kn), p.err, p.timeout_ns));
              if (!ok) break;
              k_next_ready = true;
            }
            ok = __all_sync(0xffffffffu, mbar_wait(bar(C::bSRead + t), g & 1u, p.err,
                                                   p.timeout_ns));
            if (!ok) break;
            tc_fence_after();
            issue_s_half(t, g + 1, C::k_slot(kn), 1);
          }
          ok = __all_sync(0xffffffffu, mbar_wait(bar(C::bPHalf + t), g & 1u, p.err,
                                                 p.timeout_ns));
          if (!ok) break;
          tc_fence_after();
          issue_pv_half(t, g, C::v_slot(vn), n == 0, 0);
          ok = __all_sync(0xffffffffu, mbar_wait(bar(C::bPFull + t), g & 1u, p.err,
                                                 p.timeout_ns));
          if (!ok) break;
          tc_fence_after();
          issue_pv_half(t, g, C::v_slot(vn), n == 0, 1);
          tc_commit_elect(bar(C::bOFull + t));
          if (t == last_t) tc_commit_elect(bar(C::bVEmpty + C::v_slot(vn)));
          if (more && !C::kSepP) {
            if (C::kSplitS) {
              issue_s_half(t, g + 1, C::k_slot(kn), 0);
              tc_commit_elect(bar(C::bSFull + t));
            } else {
              if (!k_next_ready) {
                ok = __all_sync(0xffffffffu, mbar_wait(bar(C::bKFull + C::k_slot(kn)),
                                                       C::k_par(kn), p.err, p.timeout_ns));
                if (!ok) break;
                tc_fence_after();
                k_next_ready = true;
              }
              issue_s(t, g + 1, C::k_slot(kn));  // commits the S barrier itself
            }
            if (n + 1 == nb - 1) tc_commit_elect(bar(C::bQEmpty + t));
            if (t == last_t) tc_commit_elect(bar(C::bKEmpty + C::k_slot(kn)));
          }
          continue;
        }
        ok = __all_sync(0xffffffffu, mbar_wait(bar(C::bPFull + t * C::NS + g % C::NS), (g / C::NS) & 1u, p.err,
                       p.timeout_ns));
        if (!ok) break;
        tc_fence_after();
        issue_pv(t, g, C::v_slot(vn), n == 0);
        if (t == last_t) tc_commit_elect(bar(C::bVEmpty + C::v_slot(vn)));
        if (C::NS == 1 && n + 1 < nb) {
          if (t == 0) {
            ok = __all_sync(0xffffffffu, mbar_wait(bar(C::bKFull + C::k_slot(kn)), C::k_par(kn), p.err,
                           p.timeout_ns));
            if (!ok) break;
            tc_fence_after();
          }
          issue_s(t, g + 1, C::k_slot(kn));
          if (n + 1 == nb - 1) tc_commit_elect(bar(C::bQEmpty + t));
          if (t == last_t) tc_commit_elect(bar(C::bKEmpty + C::k_slot(kn)));
        }
      }
    }
    k_cnt += nb;
    v_cnt += nb;
#pragma unroll
    for (int t = 0; t < C::NQ; ++t) {
      if (!(U.active >> t & 1u)) continue;
      s_cnt[t] += nb;
      ++u_cnt[t];
    }
  }
  // Wait for every MMA this thread issued before tensor memory is released.
  tc_commit_elect(bar(C::bDrain));
  mbar_wait_drain(bar(C::bDrain), 0, ok ? p.timeout_ns : 200000000ull);
}

// ---------------------------------------------------------------------------
// softmax / correction / epilogue warpgroup (one per Q tile)
// ---------------------------------------------------------------------------
// Relative bias of one 64-column half of a KV tile, for the calling thread's
// own row.
//
// Column c of the half (c = 0..63) sits at distance d = lo + 63 - c from the
// row's diagonal, where lo is the smallest distance the half meets; its bias
// is rel_bias[row][d] for 0 <= d < R and 0 elsewhere.  The thread reads the
// 9 sixteen-byte pieces [a, a + 72) with a = lo rounded down to a multiple of
// 8, which cover [lo, lo + 63].  R and a are multiples of 8, so a piece lies
// wholly inside or wholly outside [0, R); pieces outside are not read and
// count as zero.  The values then sit (lo - a) elements off the word grid
// and in reverse column order: two select stages shift by whole words and a
// byte permute per column pair takes the half-word shift and the reversal.
constexpr int kBiasPieces = 9;

__device__ __forceinline__ void bias_fetch(const uint16_t *brow, int lo, int R,
                                           uint4 (&v)[kBiasPieces]) {
  const int a = lo & ~7;
  // one base address (possibly outside the row; only in-range pieces are
  // dereferenced), pieces at immediate offsets from it
  const uint4 *src = reinterpret_cast<const uint4 *>(brow) + (a >> 3);
  const unsigned lim = brow != nullptr ? (unsigned)(R - 8) : 0u;
  const unsigned ua = brow != nullptr ? (unsigned)a : ~0u;
#pragma unroll
  for (int m = 0; m < kBiasPieces; ++m)
    v[m] = (ua + 8u * m <= lim) ? ldg_v4(src + m) : make_uint4(0u, 0u, 0u, 0u);
}

// x[c] += bias(c) * inv_scale for the 64 columns of the half (sh = lo & 7).
template <bool kHalf>
__device__ __forceinline__ void bias_apply(const uint4 (&v)[kBiasPieces], int sh,
                                           float inv_scale, float (&x)[64]) {
  uint32_t w[4 * kBiasPieces];
#pragma unroll
  for (int m = 0; m < kBiasPieces; ++m) {
    w[4 * m] = v[m].x;
    w[4 * m + 1] = v[m].y;
    w[4 * m + 2] = v[m].z;
    w[4 * m + 3] = v[m].w;
  }
  const int sw = sh >> 1;  // whole-word shift, 0..3
#pragma unroll
  for (int j = 0; j < 34; ++j) w[j] = (sw & 2) ? w[j + 2] : w[j];
#pragma unroll
  for (int j = 0; j < 33; ++j) w[j] = (sw & 1) ? w[j + 1] : w[j];
  // column pair (2k, 2k+1) -> low / high half of one word
  const uint32_t sel = (sh & 1) ? 0x3254u : 0x1032u;
  const uint64_t isc = f2(inv_scale, inv_scale);
#pragma unroll
  for (int k = 0; k < 32; ++k) {
    const uint32_t pw = __byte_perm(w[31 - k], w[32 - k], sel);
    f2_split(ffma2(f2(lo_f<kHalf>(pw), hi_f<kHalf>(pw)), isc, f2(x[2 * k], x[2 * k + 1])),
             x[2 * k], x[2 * k + 1]);
  }
}

// t: this warpgroup's Q tile among the CTA's (its tensor-memory columns and
// barriers); trow: that tile's index among the unit's tiles (its rows).  In
// the paired-SM kernel each CTA holds tile t = 0 of the unit's tile `trow`
// (its rank in the pair), and the arrivals the MMA issuer waits for (P
// ready, O free) go to the barriers of the pair's even CTA.
template <class C>
__device__ __forceinline__ void role_softmax(const FwdParams &p, uint32_t sb, uint32_t tmem,
                                             int t, int trow) {
  auto bar = [&](int i) { return sb + C::kBarOff + 8u * i; };
  auto arrive_mma = [&](int i) {
    if constexpr (C::k2SM)
      mbar_arrive_cluster(mapa_cluster(bar(i), 0));
    else
      mbar_arrive(bar(i));
  };
  constexpr int BN = C::BN, NS = C::NS;
  // row pitch of the output: the tensors' head dim (the kernel's D, or less:
  // the padding columns are never stored)
  const int dO = p.d_out;
  const int tid = static_cast<int>(threadIdx.x) - 128 * (t + 1);  // tile row == TMEM lane
  const int lane = tid & 31;
  const uint32_t lane_addr = static_cast<uint32_t>(tid & ~31) << 16;
  const float sl2 = p.scale_log2;
  uint32_t s_cnt = 0;
  bool ok = true;

  uint32_t ucnt = 0;
  Unit U;
  while (ok && next_unit<C>(p, sb, ucnt, U, ok, true)) {
    // a pair computes both of its tiles' scores in every MMA: a tile without
    // rows still takes part (its rows are invalid and never stored)
    if (!C::k2SM && !(U.active >> trow & 1u)) continue;
    const int row = U.row0 + trow * kBM + tid;
    const int i = row >> p.lgP;
    const int h = U.hq0 + (row & (p.P - 1));
    const bool valid = i < U.q_len;
    const bool warp_on = __any_sync(0xffffffffu, valid);
    const int nb = U.nb;
    // per-row constants relative to the unit's first key kv_lo, so that the
    // unit record can die before the KV loop
    // admitted keys of this row, relative to kv_lo: [st_rel, lim_rel)
    const int lim_rel = (p.wr >= 0 ? min(U.kv_hi, i + U.delta + p.wr + 1) : U.kv_hi) - U.kv_lo;
    const int st_rel = (C::MODS && p.wl >= 0) ? max(0, i + U.delta - p.wl - U.kv_lo) : 0;
    const int base0 = i + U.delta - U.kv_lo;  // distance of column 0 of tile 0
    const size_t orow = (size_t)(U.q_start + i) * p.Hq + h;  // packed (token, head) row
    void *out_row;
    float *lse_ptr;
    if constexpr (C::PARTIAL) {
      const size_t prow = (size_t)U.split * p.total_q * p.Hq + orow;
      out_row = p.o_part + prow * dO;
      lse_ptr = p.lse_part + prow;
    } else {
      out_row = reinterpret_cast<uint16_t *>(p.out) + orow * dO;
      lse_ptr = p.lse == nullptr ? nullptr
                : p.lse + (p.lse_dense ? ((size_t)U.b * p.Hq + h) * p.Sq + i
                                       : (size_t)h * p.total_q + U.q_start + i);
    }
    // the three-tile kernels serve problems without a relative bias
    const bool has_bias = C::NQ != 3 && p.rel_bias != nullptr;
    const uint16_t *brow = nullptr;
    if (has_bias && valid) brow = p.rel_bias + orow * p.R;
    float m_ref = -INFINITY, l = 0.f;
    for (int n = 0; n < nb; ++n) {
      const uint32_t g = s_cnt + n;
      const uint32_t buf = g % NS;
      const int jrel = n * BN;
      const int base = base0 - jrel;  // distance of column 0
      // does any row of this warp meet the bias band in this KV tile?
      // (three-tile kernels: every tile, so that a row never holds more
      // than half of its scores)
      const bool bias_blk = C::NQ == 3 || __any_sync(0xffffffffu, has_bias && valid && base >= 0 &&
                                                                      base - (BN - 1) < p.R);
      const uint32_t s_addr = tmem + lane_addr + C::s_col(t, buf);
      const uint32_t p_addr = tmem + lane_addr + C::p_col(t, buf);
      const int lim_c = lim_rel - jrel;  // columns at or past lim_c are masked
      const int st_c = C::MODS ? st_rel - jrel : 0;  // and columns before st_c
      // no row of the warp has a masked column here: the FMA-pipe exponential
      // may stand in for some of the MUFU ones
      const bool poly_ok = __all_sync(0xffffffffu, lim_c >= BN && st_c <= 0);
      // one arrival per warp, after this thread's tensor-memory accesses
      auto warp_arrive = [&](int b) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) arrive_mma(b);
      };
      auto wait_scores = [&]() -> bool {
        const bool w = __all_sync(0xffffffffu,
                                  mbar_wait(bar(C::bSFull + t * NS + buf), (g / NS) & 1u,
                                            p.err, p.timeout_ns));
        tc_fence_after();
        return w;
      };
      // O (and l) rescale by f once the running max has moved; for n > 0
        // the previous P.V must have completed (guaranteed by the score
        // barrier when S is single-buffered, waited for otherwise).
        auto rescale_o = [&](float f) -> bool {
          if (NS == 2 || C::kSepP) {
            const uint32_t gp = g - 1;
            if (!__all_sync(0xffffffffu, mbar_wait(bar(C::bOFull + t * NS + gp % NS),
                                                   (gp / NS) & 1u, p.err, p.timeout_ns)))
              return false;
            tc_fence_after();
          }
          const uint32_t o_addr = tmem + lane_addr + C::o_col(t);
#pragma unroll 1
          for (int c = 0; c < C::kOStride / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(o_addr + 32 * c, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
            tmem_st32(o_addr + 32 * c, o);
          }
          return true;
        };
      // separate P buffer: P(g-1).V must be done before P(g) overwrites it
      auto wait_prev_pv = [&]() -> bool {
        const uint32_t gp = g - 1;
        const bool w = __all_sync(0xffffffffu, mbar_wait(bar(C::bOFull + t * NS + gp % NS),
                                                         (gp / NS) & 1u, p.err,
                                                         p.timeout_ns));
        tc_fence_after();
        return w;
      };
      // The two kinds of tile take disjoint paths (each with its own wait) so
      // that their register-resident arrays never meet at a join.
      if (bias_blk) {
        // Tiles that meet the bias band: 64-column halves, each with its own
        // running-max update (online softmax at half-tile granularity), so
        // that a half's bias and its scores fit in registers together.  With
        // conditional rescaling the second half rarely moves the reference
        // max; when it does, the first half's P (already in tensor memory) is
        // rescaled along with O and l.  A half's bias loads are in flight
        // while the thread waits for the scores (first half) or works on the
        // half before it.
        const int lo0 = base - 63;  // smallest distance met by half 0
        const int bsh = lo0 & 7;    // misalignment, the same for every half of the row
        auto half_on = [&](int lo) {  // some row of the warp meets the band in this half
          return __any_sync(0xffffffffu, brow != nullptr && lo + 63 >= 0 && lo < p.R);
        };
        uint4 bv[kBiasPieces];
        bool bon = C::NQ != 3 && half_on(lo0);
        if (bon) bias_fetch(brow, lo0, p.R, bv);
        ok = wait_scores();
        if (!ok) break;
        if (warp_on) {
#pragma unroll
          for (int hf = 0; hf < BN / 64; ++hf) {
            float x[64];
            {
              uint32_t r0[32], r1[32];
              tmem_ld32(s_addr + 64 * hf, r0);
              tmem_ld32(s_addr + 64 * hf + 32, r1);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) {
                x[e] = __uint_as_float(r0[e]);
                x[32 + e] = __uint_as_float(r1[e]);
              }
            }
            // every score read: the next tile's upper keys may land
            if ((C::kSplitS || C::kSepP) && hf == BN / 64 - 1) warp_arrive(C::bSRead + t);
            if constexpr (C::MODS) {
              if (p.cap_a > 0.f) softcap_all<64>(x, p.cap_a, p.cap_b);
            }
            if (bon) bias_apply<C::HALF>(bv, bsh, p.inv_scale, x);
            if (hf + 1 < BN / 64) {
              const int lo = lo0 - 64 * (hf + 1);
              bon = C::NQ != 3 && half_on(lo);
              if (bon) bias_fetch(brow, lo, p.R, bv);
            }
            if (lim_c < 64 * hf + 64 || st_c > 64 * hf) {
#pragma unroll
              for (int e = 0; e < 64; ++e)
                if (64 * hf + e >= lim_c || 64 * hf + e < st_c) x[e] = -INFINITY;
            }
          // running-max update with conditional rescaling
          const float m_new = fmaxf(m_ref, row_max<0, 64>(x));
          if (n == 0 && hf == 0) {
            m_ref = m_new;
          } else {
            const bool need_rs = (m_new - m_ref) > p.thr_raw;
            if (__any_sync(0xffffffffu, need_rs)) {
              const float f = need_rs ? ex2_approx((m_ref - m_new) * sl2) : 1.f;
              if (need_rs) {
                l *= f;
                m_ref = m_new;
              }
              if (n > 0) {
                ok = rescale_o(f);
                if (!ok) break;
              }
              if (hf > 0) {  // P of the earlier halves of this tile
#pragma unroll 1
                for (int c = 0; c < hf; ++c) {
                  uint32_t o[32];
                  tmem_ld32(p_addr + 32 * c, o);
                  tmem_wait_ld();
#pragma unroll
                  for (int e = 0; e < 32; ++e)
                    o[e] = pack2<C::HALF>(lo_f<C::HALF>(o[e]) * f, hi_f<C::HALF>(o[e]) * f);
                  tmem_st32(p_addr + 32 * c, o);
                }
              }
              tmem_wait_st();
            }
          }
          const float mc = (m_ref == -INFINITY) ? 0.f : m_ref * sl2;
          uint32_t pk[32];
          if (kPolyPairs > 0 && poly_ok)
            l += exp_pack<C::HALF, true, 0, 64>(x, sl2, mc, pk);
          else
            l += exp_pack<C::HALF, false, 0, 64>(x, sl2, mc, pk);
          // P half hf -> columns [32 hf, 32 hf + 32): only score columns
          // already read are overwritten (or the separate P buffer's)
          if (C::kSepP && hf == 0 && n > 0) {
            ok = wait_prev_pv();
            if (!ok) break;
          }
          tmem_st32(p_addr + 32 * hf, pk);
          }
          if (!ok) break;
          tmem_wait_st();
        } else {
          if (C::kSplitS || C::kSepP) warp_arrive(C::bSRead + t);
          // A warp without rows must not run ahead: with a separate P buffer
          // S(g+1) is ready while the other warps still work on tile g, and
          // its P arrivals for g+1 would complete their phase for g.  Its
          // arrivals for tile g wait until P(g-1).V is done, i.e. until every
          // warp has finished tile g-1.
          if (C::kSepP && n > 0) {
            ok = wait_prev_pv();
            if (!ok) break;
          }
        }
        // the bias path may rescale its first P half after storing it, so the
        // first-half signal waits for the whole tile
        if (C::kSplitPV) warp_arrive(C::bPHalf + t);
        warp_arrive(C::bPFull + t * NS + buf);
      } else {
        ok = wait_scores();
        if (!ok) break;
        if (warp_on) {
          // Tiles without bias: the whole row of scores in registers, one
          // running-max update per tile.
          float s[BN];
#pragma unroll
          for (int c = 0; c < BN / 32; ++c) {
            uint32_t r[32];
            tmem_ld32(s_addr + 32 * c, r);
#pragma unroll
            for (int e = 0; e < 32; ++e) s[32 * c + e] = __uint_as_float(r[e]);
          }
          tmem_wait_ld();
          if (C::kSplitS || C::kSepP) warp_arrive(C::bSRead + t);
          if constexpr (C::MODS) {
            if (p.cap_a > 0.f) softcap_all<BN>(s, p.cap_a, p.cap_b);
          }
          if (lim_c < BN || st_c > 0) {
#pragma unroll
            for (int c = 0; c < BN; ++c)
              if (c >= lim_c || c < st_c) s[c] = -INFINITY;
          }
          const float m_new = fmaxf(m_ref, row_max<0, BN>(s));
          if (n == 0) {
            m_ref = m_new;
          } else {
            const bool need_rs = (m_new - m_ref) > p.thr_raw;
            if (__any_sync(0xffffffffu, need_rs)) {
              const float f = need_rs ? ex2_approx((m_ref - m_new) * sl2) : 1.f;
              if (need_rs) {
                l *= f;
                m_ref = m_new;
              }
              ok = rescale_o(f);
              if (!ok) break;
              tmem_wait_st();
            }
          }
          const float mc = (m_ref == -INFINITY) ? 0.f : m_ref * sl2;
          {
            uint32_t pk[32];
            if (kPolyPairs > 0 && poly_ok)
              l += exp_pack<C::HALF, true, 0, 64>(s, sl2, mc, pk);
            else
              l += exp_pack<C::HALF, false, 0, 64>(s, sl2, mc, pk);
            if (C::kSepP && n > 0) {
              ok = wait_prev_pv();
              if (!ok) break;
            }
            tmem_st32(p_addr, pk);
            if (C::kSplitPV) {
              tmem_wait_st();
              warp_arrive(C::bPHalf + t);
            }
          }
          if constexpr (BN == 128) {
            uint32_t pk[32];
            if (kPolyPairs > 0 && poly_ok)
              l += exp_pack<C::HALF, true, 64, 64>(s, sl2, mc, pk);
            else
              l += exp_pack<C::HALF, false, 64, 64>(s, sl2, mc, pk);
            tmem_st32(p_addr + 32, pk);
          }
          tmem_wait_st();
          warp_arrive(C::bPFull + t * NS + buf);
        } else {
          if (C::kSplitS || C::kSepP) warp_arrive(C::bSRead + t);
          if (C::kSepP && n > 0) {  // no running ahead (see the bias path)
            ok = wait_prev_pv();
            if (!ok) break;
          }
          if (C::kSplitPV) warp_arrive(C::bPHalf + t);
          warp_arrive(C::bPFull + t * NS + buf);
        }
      }
    }
    if (!ok) break;

    // epilogue
    const float inv_l = l > 0.f ? 1.f / l : 0.f;
    const float lse_v = l > 0.f ? (m_ref * sl2 + lg2_approx(l)) * 0.69314718055994531f : -INFINITY;
    if (nb > 0) {
      const uint32_t gl = s_cnt + nb - 1;
      ok = __all_sync(0xffffffffu, mbar_wait(bar(C::bOFull + t * NS + gl % NS), (gl / NS) & 1u,
                                             p.err, p.timeout_ns));
      if (!ok) break;
      tc_fence_after();
    }
    if (warp_on) {
#pragma unroll 1
      for (int c = 0; c < C::kOStride / 32; ++c) {
        uint32_t r[32];
        if (nb > 0) {
          tmem_ld32(tmem + lane_addr + C::o_col(t) + 32 * c, r);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) r[e] = 0u;
        }
        if (valid) {
          if constexpr (C::PARTIAL) {
            float *dst = reinterpret_cast<float *>(out_row) + 32 * c;
            if (p.st32) {  // 8 columns per 32-byte store
#pragma unroll
              for (int e = 0; e < 32; e += 8) {
                if (32 * c + e >= dO) break;
                uint4 a, b;
                a.x = __float_as_uint(__uint_as_float(r[e]) * inv_l);
                a.y = __float_as_uint(__uint_as_float(r[e + 1]) * inv_l);
                a.z = __float_as_uint(__uint_as_float(r[e + 2]) * inv_l);
                a.w = __float_as_uint(__uint_as_float(r[e + 3]) * inv_l);
                b.x = __float_as_uint(__uint_as_float(r[e + 4]) * inv_l);
                b.y = __float_as_uint(__uint_as_float(r[e + 5]) * inv_l);
                b.z = __float_as_uint(__uint_as_float(r[e + 6]) * inv_l);
                b.w = __float_as_uint(__uint_as_float(r[e + 7]) * inv_l);
                stg_v8(dst + e, a, b);
              }
              continue;
            }
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
              if (32 * c + e >= dO) break;
              float4 w = make_float4(__uint_as_float(r[e]) * inv_l, __uint_as_float(r[e + 1]) * inv_l,
                                     __uint_as_float(r[e + 2]) * inv_l,
                                     __uint_as_float(r[e + 3]) * inv_l);
              *reinterpret_cast<float4 *>(dst + e) = w;
            }
          } else {
            uint16_t *dst = reinterpret_cast<uint16_t *>(out_row) + 32 * c;
            if (p.st32) {  // 16 columns per 32-byte store
#pragma unroll
              for (int e = 0; e < 32; e += 16) {
                if (32 * c + e >= dO) break;
                uint4 a, b;
                a.x = pack2<C::HALF>(__uint_as_float(r[e]) * inv_l, __uint_as_float(r[e + 1]) * inv_l);
                a.y = pack2<C::HALF>(__uint_as_float(r[e + 2]) * inv_l, __uint_as_float(r[e + 3]) * inv_l);
                a.z = pack2<C::HALF>(__uint_as_float(r[e + 4]) * inv_l, __uint_as_float(r[e + 5]) * inv_l);
                a.w = pack2<C::HALF>(__uint_as_float(r[e + 6]) * inv_l, __uint_as_float(r[e + 7]) * inv_l);
                b.x = pack2<C::HALF>(__uint_as_float(r[e + 8]) * inv_l, __uint_as_float(r[e + 9]) * inv_l);
                b.y = pack2<C::HALF>(__uint_as_float(r[e + 10]) * inv_l, __uint_as_float(r[e + 11]) * inv_l);
                b.z = pack2<C::HALF>(__uint_as_float(r[e + 12]) * inv_l, __uint_as_float(r[e + 13]) * inv_l);
                b.w = pack2<C::HALF>(__uint_as_float(r[e + 14]) * inv_l, __uint_as_float(r[e + 15]) * inv_l);
                stg_v8(dst + e, a, b);
              }
              continue;
            }
#pragma unroll
            for (int e = 0; e < 32; e += 8) {
              if (32 * c + e >= dO) break;
              uint4 w;
              w.x = pack2<C::HALF>(__uint_as_float(r[e]) * inv_l, __uint_as_float(r[e + 1]) * inv_l);
              w.y = pack2<C::HALF>(__uint_as_float(r[e + 2]) * inv_l, __uint_as_float(r[e + 3]) * inv_l);
              w.z = pack2<C::HALF>(__uint_as_float(r[e + 4]) * inv_l, __uint_as_float(r[e + 5]) * inv_l);
              w.w = pack2<C::HALF>(__uint_as_float(r[e + 6]) * inv_l, __uint_as_float(r[e + 7]) * inv_l);
              *reinterpret_cast<uint4 *>(dst + e) = w;
            }
          }
        }
      }
    }
    if (valid && lse_ptr != nullptr) *lse_ptr = lse_v;
    if (nb > 0) {
      tc_fence_before();
      if constexpr (C::k2SM) {  // one arrival per warp on the even CTA's barrier
        __syncwarp();
        if (lane == 0) arrive_mma(C::bOEmpty + t);
      } else {
        mbar_arrive(bar(C::bOEmpty + t));
      }
    }
    s_cnt += nb;
  }
}

template <class C>
__global__ void __launch_bounds__(C::kThreads, 1) fa_fwd_kernel(const __grid_constant__ FwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const int warp = warp_id_sync();
  const int lane = threadIdx.x & 31;

  if (warp == 0 && lane == 0) {
    for (int b = 0; b < C::kNumBars; ++b) {
      uint32_t cnt = 1;
      if (b >= C::bPFull && b < C::bPFull + C::NQ * C::NS) cnt = 4;  // one per warp
      if (b >= C::bSRead && b < C::bPHalf + C::NQ) cnt = 4;
      if (b >= C::bOEmpty && b < C::bOEmpty + C::NQ) cnt = 128;
      if (b >= C::bUEmpty && b < C::bUEmpty + kUnitRing) cnt = C::kUnitConsumers;
      mbar_init(sb + C::kBarOff + 8u * b, cnt);
    }
    fence_mbar_init();
    tma_prefetch_desc(&p.tm_q);
    tma_prefetch_desc(&p.tm_k);
    tma_prefetch_desc(&p.tm_v);
  }
  if (warp == 1) {
    tmem_alloc(sb + C::kSlotOff, C::kTmemCols);
    tmem_relinquish();
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
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + C::kSlotOff);

  if (warp < 4) {
    if constexpr (C::kSplitRegs) regs_lower<C::kRegsCtl>();
    if (warp == 0) {
      role_producer<C>(p, sb);  // whole warp; lane 0 issues the copies
    } else if (warp == 1) {
      role_mma<C>(p, sb, tmem);  // whole warp; MMAs issued by the elected lane
    } else if (warp == 2) {
      role_scheduler<C>(p, sch, sb);  // whole warp; lane 0 publishes
    }
  } else {
    if constexpr (C::kSplitRegs) regs_raise<C::kRegsSoftmax>();
    role_softmax<C>(p, sb, tmem, warp / 4 - 1, warp / 4 - 1);
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// split-KV merge: one warp per packed (token, head) row.  F32OUT writes the
// merged O in fp32 and its LSE at the row's own index, i.e. one more partial
// in the layout the splits use (a key shard's partial, merged again later).
// ---------------------------------------------------------------------------
template <int D, bool HALF, bool F32OUT = false>
__global__ void __launch_bounds__(256) fa_combine_kernel(const float *__restrict__ o_part,
                                                         const float *__restrict__ lse_part,
                                                         int ns, long long rows, void *out,
                                                         float *lse, int Hq, int Sq,
                                                         int total_q, int lse_dense) {
  constexpr int E = D / 32;  // elements per lane
  const long long r = (long long)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  const float L2E = 1.4426950408889634f;
  float m = -INFINITY;
  for (int s = lane; s < ns; s += 32) m = fmaxf(m, lse_part[(long long)s * rows + r]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float z = 0.f;
  if (m != -INFINITY)
    for (int s = lane; s < ns; s += 32) z += ex2_approx((lse_part[(long long)s * rows + r] - m) * L2E);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
  const float Lse = (m == -INFINITY) ? -INFINITY : m + lg2_approx(z) * 0.69314718055994531f;
  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  if (m != -INFINITY) {
    // splits in groups of 8 whose loads are all issued before any is used
    // (a weight of 0 stands for a split with no keys)
    constexpr int U = 8;
    for (int s0 = 0; s0 < ns; s0 += U) {
      float w[U];
      float x[U][E];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int s = s0 + u;
        w[u] = 0.f;
        if (s < ns) {
          const float ls = __ldg(lse_part + (long long)s * rows + r);
          w[u] = ls == -INFINITY ? 0.f : ex2_approx((ls - Lse) * L2E);
          const float *src = o_part + ((long long)s * rows + r) * D + lane * E;
          if constexpr (E % 4 == 0) {
#pragma unroll
            for (int e = 0; e < E; e += 4) {
              const float4 v = __ldg(reinterpret_cast<const float4 *>(src + e));
              x[u][e] = v.x;
              x[u][e + 1] = v.y;
              x[u][e + 2] = v.z;
              x[u][e + 3] = v.w;
            }
          } else {
#pragma unroll
            for (int e = 0; e < E; e += 2) {
              const float2 v = __ldg(reinterpret_cast<const float2 *>(src + e));
              x[u][e] = v.x;
              x[u][e + 1] = v.y;
            }
          }
        } else {
#pragma unroll
          for (int e = 0; e < E; ++e) x[u][e] = 0.f;
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] += w[u] * x[u][e];
    }
  }
  if constexpr (F32OUT) {
    float *dst = reinterpret_cast<float *>(out) + r * D + lane * E;
    if constexpr (E % 4 == 0) {
#pragma unroll
      for (int e = 0; e < E; e += 4)
        *reinterpret_cast<float4 *>(dst + e) = make_float4(acc[e], acc[e + 1], acc[e + 2], acc[e + 3]);
    } else {
#pragma unroll
      for (int e = 0; e < E; e += 2)
        *reinterpret_cast<float2 *>(dst + e) = make_float2(acc[e], acc[e + 1]);
    }
    if (lane == 0) lse[r] = Lse;
    return;
  }
  uint16_t *dst = reinterpret_cast<uint16_t *>(out) + r * D + lane * E;
  if constexpr (E % 4 == 0) {
#pragma unroll
    for (int e = 0; e < E; e += 4) {
      uint2 w;
      w.x = pack2<HALF>(acc[e], acc[e + 1]);
      w.y = pack2<HALF>(acc[e + 2], acc[e + 3]);
      *reinterpret_cast<uint2 *>(dst + e) = w;
    }
  } else {
#pragma unroll
    for (int e = 0; e < E; e += 2)
      *reinterpret_cast<uint32_t *>(dst + e) = pack2<HALF>(acc[e], acc[e + 1]);
  }
  if (lane == 0 && lse != nullptr) {
    const long long tok = r / Hq;
    const int h = (int)(r % Hq);
    const long long li =
        lse_dense ? ((tok / Sq) * Hq + h) * (long long)Sq + tok % Sq : (long long)h * total_q + tok;
    lse[li] = Lse;
  }
}

// The same merge for head dims d that are not a multiple of 64 (a multiple
// of 8, at most 256): lane l handles the column pairs starting at 2l + 64k.
template <bool HALF, bool F32OUT>
__global__ void __launch_bounds__(256) fa_combine_narrow_kernel(const float *__restrict__ o_part,
                                                                const float *__restrict__ lse_part,
                                                                int ns, long long rows, int d,
                                                                void *out, float *lse, int Hq,
                                                                int Sq) {
  const long long r = (long long)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  const float L2E = 1.4426950408889634f;
  float m = -INFINITY;
  for (int s = lane; s < ns; s += 32) m = fmaxf(m, lse_part[(long long)s * rows + r]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float z = 0.f;
  if (m != -INFINITY)
    for (int s = lane; s < ns; s += 32) z += ex2_approx((lse_part[(long long)s * rows + r] - m) * L2E);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
  const float Lse = (m == -INFINITY) ? -INFINITY : m + lg2_approx(z) * 0.69314718055994531f;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  if (m != -INFINITY) {
    for (int s = 0; s < ns; ++s) {
      const float ls = __ldg(lse_part + (long long)s * rows + r);
      if (ls == -INFINITY) continue;
      const float w = ex2_approx((ls - Lse) * L2E);
      const float *src = o_part + ((long long)s * rows + r) * d;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int c = 2 * lane + 64 * k;
        if (c < d) {
          const float2 v = __ldg(reinterpret_cast<const float2 *>(src + c));
          acc[2 * k] += w * v.x;
          acc[2 * k + 1] += w * v.y;
        }
      }
    }
  }
  if constexpr (F32OUT) {
    float *dst = reinterpret_cast<float *>(out) + r * d;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int c = 2 * lane + 64 * k;
      if (c < d) *reinterpret_cast<float2 *>(dst + c) = make_float2(acc[2 * k], acc[2 * k + 1]);
    }
    if (lane == 0) lse[r] = Lse;
  } else {
    uint16_t *dst = reinterpret_cast<uint16_t *>(out) + r * d;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int c = 2 * lane + 64 * k;
      if (c < d) *reinterpret_cast<uint32_t *>(dst + c) = pack2<HALF>(acc[2 * k], acc[2 * k + 1]);
    }
    if (lane == 0 && lse != nullptr) {
      const long long tok = r / Hq;
      const int h = (int)(r % Hq);
      lse[((tok / Sq) * Hq + h) * (long long)Sq + tok % Sq] = Lse;
    }
  }
}

}  // namespace fab
