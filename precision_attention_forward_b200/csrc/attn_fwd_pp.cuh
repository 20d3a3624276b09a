// attn_fwd_pp.cuh -- MXFP8 attention forward over pairs of query tiles.
//
// Computes, per (sequence, head), O = softmax(Q K^T * qd * kd / sqrt(128)) V * vd and the
// natural-log LSE for noncausal head_dim 128 over packed variable-length sequences (LP-FA4 README,
// "MXFP8 forward and backward"). Q and K are MXFP8 (E4M3 payload, one E8M0 scale per 32 elements
// along head_dim). PV modes: bf16 (V MXFP8, dequantized exactly to BF16 in shared memory, P
// rounded to BF16), BF16 V input (V given in BF16, P rounded to BF16), fp8 (V an unscaled E4M3 cast,
// implicit dequant scale 1.0, P rounded to E4M3; FastVideo #1654 "fp8 PV mode for the FA4-FP4
// attention path") and block-scaled MXFP8 (P and V scaled per 32 keys). O is BF16; absent
// descales are the literal 1.0f on the same code path (vLLM #63232, "Claims").
//
// Work unit: two consecutive 128-row query tiles Q0, Q1 of one (sequence, head) -- the second
// absent when the sequence has an odd number of tiles and this is its last -- against all K/V
// tiles of that sequence. Each softmax warpgroup owns one query tile: its own row reference, its
// own row sums and its own O accumulator, so nothing of the online softmax crosses warpgroups
// (FlashAttention-4's two-tile ping-pong). Every K and V tile loaded serves both query tiles.
//
// At a unit boundary the softmax warps only hand their row normalisers to the epilogue warps and
// go on; with bf16 P they also have the next unit's description decoded ahead, and the producer
// (one Q stage) has prefetched the next unit's Q tiles into L2.
//
// Warp roles (512 threads):
//   warp 0        Q/K producer: Q0, Q1 and their scale atoms once per unit, then K tiles + atoms.
//   warp 3        V producer: V tiles (+ scale atoms for MXFP8 V; BF16 V as two swizzled boxes).
//   warp 1        TMEM owner and QK issuer: S = Q_i K_j^T (tcgen05.mma kind::mxf8f6f4.block_scale,
//                 M128 N128 K128) into the one S buffer, for i = 0, 1 in turn, each as soon as the
//                 previous S has been read out by its warpgroup.
//   warp 2        PV issuer: O_i += P V_j -- kind::f8f6f4 or kind::mxf8f6f4.block_scale with P in
//                 TMEM (8-bit P), kind::f16 with P and BF16 V in shared memory (bf16 P).
//   warps 4..7    softmax of Q0; warps 8..11 softmax of Q1 (one thread per query row).
//   warps 12..15  bf16 PV with MXFP8 V converted in the kernel: convert V tiles to BF16 in shared
//                 memory (the softmax warps then write O themselves); every other mode: epilogue,
//                 i.e. read each finished O_i from TMEM, scale, store BF16 O and the LSE, while the
//                 softmax warps go on with the next unit.
//
// TMEM (512 columns): S [0, 128); O_i [128 + 128 i, 256 + 128 i); 8-bit P in three slots
// [384 + 32 slot, +32); scale atoms after them (see the column constants). A single S buffer is what
// makes room for the block-scaled QK's scale factors next to two O accumulators; the warpgroups
// pass it back and forth, and P has room of its own (TMEM slots, or shared memory for bf16 P), so a
// warpgroup's next S can be computed while its exponentials of the previous tile still run.
#pragma once

#include "attn_fwd.cuh"

namespace lpfa {
namespace pp {

// LPFA_PP_EPI_WG: warps 12..15 write O and the LSE in the modes where they convert no V (else the
// softmax warps do, after each unit).
#ifndef LPFA_PP_EPI_WG
#define LPFA_PP_EPI_WG 1
#endif

// LPFA_PP_BF_P_SMEM: bf16 P in two shared-memory slots (PV as a shared-memory MMA), else in one
// 64-column TMEM slot that the two warpgroups use in turn. Two slots decouple the warpgroups; the
// single TMEM slot reads less shared memory and leaves room for two Q stages. (Measured: the
// shared-memory slots are faster on most workloads.)
#ifndef LPFA_PP_BF_P_SMEM
#define LPFA_PP_BF_P_SMEM 1
#endif
constexpr bool kBfPSmem = LPFA_PP_BF_P_SMEM != 0;

// P tiles rotate through slots in the order the PV products consume them (tile j of a unit: query
// tile 0, then 1): three 32-column TMEM slots for 8-bit P, so a softmax warpgroup storing P waits
// only for the PV three P tiles back; for bf16 P two 32 KB shared-memory slots, or one 64-column
// TMEM slot (all the columns there are) written by the two warpgroups in turn.
constexpr uint32_t kPSlots = 3;
constexpr uint32_t kPSlotsBf = kBfPSmem ? 2 : 1;
constexpr uint32_t kColS = 0;
constexpr uint32_t kColO = 128;    // + 128 * i
constexpr uint32_t kColP = 384;    // + 32 * slot (8-bit P); bf16 P: [384, 448)
// Scale atoms. fp8 PV and bf16 PV: the Q atoms of both tiles per unit stage and the K atoms in two
// slots, all copied into TMEM ahead of the QK that reads them. MXFP8 PV (whose P and V atoms take
// the rest of the columns): one Q and one K slot, copied right before each QK, once the previous
// QK -- the slots' last reader -- is known to have completed.
constexpr uint32_t kColSFA8 = 480;   // + 8 * qstage + 4 * i   (fp8 PV)
constexpr uint32_t kColSFB8 = 496;   // + 4 * (kc & 1)         (fp8 PV)
constexpr uint32_t kColSFABf = kBfPSmem ? 384 : 448;  // + 8 * qstage + 4 * i   (bf16 PV)
constexpr uint32_t kColSFBBf = kBfPSmem ? 400 : 464;  // + 4 * (kc & 1)         (bf16 PV)
constexpr uint32_t kColSFA = 480;    // Q scale atom of the QK being issued (MXFP8 PV)
constexpr uint32_t kColSFB = 484;    // K scale atom of the current K tile (MXFP8 PV)
constexpr uint32_t kColSFP = 488;    // + 4 * slot: P scale atom (MXFP8 PV)
constexpr uint32_t kColSFV = 500;    // + 4 * (vc % 3): V scale atom (MXFP8 PV)
static_assert(kColP + 32 * kPSlots <= kColSFA && kColSFB8 + 8 <= kTmemCols && kColSFV + 4 * 3 <= kTmemCols &&
              (kBfPSmem ? kColO + 256 : kColP + 64) <= kColSFABf && kColSFBBf + 8 <= kTmemCols, "TMEM columns");

constexpr uint32_t kBfTileBytes = 128 * 128 * 2;  // 128 keys x 128 BF16 (two 64-column swizzle atoms)
constexpr uint32_t kBfAtomBytes = 128 * 128;      // one 128-row x 128-byte swizzle atom

// Shared memory (offsets from a 1024-byte aligned base) and ring depths per PV mode. The bf16 P
// modes keep BF16 V tiles (32 KB each) in shared memory, and with P there too (two 32 KB slots)
// their Q has one stage and their V rings are shallower.
constexpr int kSchedSplit = 2 + 2 * kMaxSortSeqs + 1;      // units before the split tail
constexpr int kSchedMeta = kSchedSplit + 1;                // first metadata copy in sched[]
constexpr int kSchedInts = kSchedMeta + 4 * (kMaxSortSeqs + 1);

template <int kPv>
struct Smem {
  static constexpr bool kBf = kPv == kPvBf16Mx || kPv == kPvBf16In;  // bf16 P, BF16 V
  static constexpr bool kVIn = kPv == kPvBf16In;                     // BF16 V input
  static constexpr bool kPS_ = kBf && kBfPSmem;                      // bf16 P in shared memory
  static constexpr int kQS = kPS_ ? 1 : kQStages;                     // Q stages (two tiles each)
  static constexpr int kKS = kBf ? 3 : 5;                             // K ring
  static constexpr int kVS = kVIn ? 0 : (kBf ? 2 : 4);                // 8-bit V ring
  static constexpr int kVBS = kBf ? (kPS_ ? (kVIn ? 2 : 1) : (kVIn ? 3 : 2)) : 0;  // BF16 V ring
  static constexpr int kPS = kPS_ ? static_cast<int>(kPSlotsBf) : 0;  // bf16 P slots in shared memory
  static constexpr bool kVsf = kPv == kPvMx || kPv == kPvBf16Mx;     // V tiles come with a scale atom
  static constexpr uint32_t q = 0;
  static constexpr uint32_t k = q + kQS * 2 * kTileBytes;
  static constexpr uint32_t v = k + kKS * kTileBytes;
  static constexpr uint32_t vbf = v + kVS * kTileBytes;
  static constexpr uint32_t pbf = vbf + kVBS * kBfTileBytes;
  static constexpr uint32_t q_sf = pbf + kPS * kBfTileBytes;               // [kQS][2] atoms
  static constexpr uint32_t k_sf = q_sf + kQS * 2 * kAtomBytes;
  static constexpr uint32_t v_sf = k_sf + kKS * kAtomBytes;                // MXFP8 V only
  static constexpr uint32_t p_sf = v_sf + (kVsf ? kVS * kAtomBytes : 0u);  // [kPSlots] P atoms (MXFP8 PV)
  static constexpr uint32_t sched = p_sf + (kPv == kPvMx ? kPSlots * kAtomBytes : 0u);  // n, units, order, prefix
  static constexpr uint32_t bars = sched + ((kSchedInts * 4) + 15) / 16 * 16;
  static constexpr uint32_t num_bars = 56;
  static constexpr uint32_t misc = bars + num_bars * 8;                     // tmem base, abort flag
  static constexpr uint32_t stats = misc + 64;                              // [2][128] (O scale, LSE)
  static constexpr uint32_t total = stats + 2 * 128 * 8;
  static_assert(kKS <= 6 && kVS <= 6 && kVBS <= 3, "ring barriers");
};
template <int kPv> constexpr uint32_t smem_bytes() { return Smem<kPv>::total + 1024; }
static_assert(smem_bytes<kPvFp8>() <= 227 * 1024 && smem_bytes<kPvMx>() <= 227 * 1024 &&
              smem_bytes<kPvBf16Mx>() <= 227 * 1024 && smem_bytes<kPvBf16In>() <= 227 * 1024, "shared memory");

enum Bar : int {
  kBarQFull = 0, kBarQEmpty = 2,     // [kQStages]
  kBarKFull = 4, kBarKEmpty = 10,    // [kKStages <= 6]
  kBarVFull = 16, kBarVEmpty = 22,   // [kVStages <= 6]
  kBarSFull = 28,   // [i] S computed for warpgroup i            (MMA commit)
  kBarSFree = 30,   // S read out by the warpgroup it was for     (4 warps)
  kBarPReady = 31,  // [slot] P stored, O rescaled if needed      (4 warps)
  kBarPVDone = 34,  // [slot] the PV reading the slot complete   (MMA commit)
  kBarOFull = 37,   // [i] every PV_i of the unit complete        (MMA commit)
  kBarOEmpty = 39,  // [i] O_i read out by the epilogue           (4 warps)
  kBarDrain = 41,   // QK issuer's own tcgen05 work done
  kBarDrainPV = 42, // PV issuer's own tcgen05 work done
  kBarVbfFull = 43, // [3] BF16 V tile in shared memory (TMA, or the 4 converter warps)
  kBarVbfEmpty = 46, // [3] the PVs reading the BF16 V tile complete (MMA commit)
  kBarStatsFull = 49, // [i] warpgroup i's row normalisers and LSE in shared memory (4 warps)
  kBarStatsFree = 51, // [i] the epilogue warpgroup has read them                 (4 warps)
  kBarCount = 53
};
static_assert(kBarCount <= Smem<kPvFp8>::num_bars, "barrier array");

// Diagnostic sites (g_lpfa_status[1]) of this kernel's waits: 100 + the role's step.
enum PairSite : int {
  kPSiteProducerQ = 101, kPSiteProducerK, kPSiteProducerV, kPSiteMmaQ, kPSiteMmaK, kPSiteMmaS, kPSiteMmaP,
  kPSiteMmaO, kPSiteMmaV, kPSiteSoftS, kPSiteSoftPV, kPSiteSoftO, kPSiteDrain, kPSiteDebugStall, kPSiteTmem,
  kPSiteConvV, kPSiteConvE, kPSiteEpiO, kPSiteEpiStats, kPSiteSoftStats
};

// A work unit: query tiles qtile0 and (has_q1) qtile0 + 1 of one (sequence, head). seq is the
// key/value sequence (and the descales' sequence index); q_row0 the first query row read, o_row0
// the first output (and LSE) row written -- they differ only for a shared query set.
struct PairUnit {
  int h, seq, qtile0, q_row0, o_row0, q_len, k_row0, k_len, nkv, sbq, sbk, has_q1;
};

// Unit order in shared memory: sched[0] = n, sched[1] = number of units, then order[kMaxSortSeqs],
// prefix[kMaxSortSeqs + 1] and (n > 0) copies of the metadata the units are decoded from:
// cu_q, scale_off_q, cu_k, scale_off_k, kMaxSortSeqs + 1 entries each, so that decoding a unit
// reads only shared memory. When the pair units would leave a last partial wave of r units with
// 2 r <= the grid size, those r pairs (the shortest, at the end of the longest-first order) are split
// into 2 r single-tile units, one per CTA, instead of r CTAs running a whole pair while the rest
// wait: sched[kSchedSplit] is the number of units before the split tail. A single-tile unit that
// would be the absent second tile of a pair has nkv = -1 and is skipped by every role. For 1 <= n <= kMaxSortSeqs sequences the units are pairs of query
// tiles: sequences by decreasing key-tile count (longest first), each taking heads * ceil(tiles / 2)
// consecutive units, pairs innermost, so that the CTAs running together share one (sequence,
// head)'s K/V through L2 and the static round-robin over the list approximates longest-processing-
// time scheduling. Beyond kMaxSortSeqs sequences (n = 0) every unit is a single tile in the packed
// head-major order (the pairs' prefix would not fit in shared memory); with a shared query set
// (n = -1) every key/value sequence has the same number of query tiles, so pairs stay and the
// plain order (sequence, head, pair) needs no prefix.
__device__ __forceinline__ int query_tiles_of(const AttnParams& p, int seq) {
  const int qs = p.shared_q ? 0 : seq;
  return __ldg(p.so_q + qs + 1) - __ldg(p.so_q + qs);
}

__device__ __forceinline__ void build_pair_order(const AttnParams& p, int* sched) {
  const int n = p.num_seqs;
  int* s_order = sched + 2;
  int* s_pre = sched + 2 + kMaxSortSeqs;
  if (n > kMaxSortSeqs) {
    if (threadIdx.x == 0) {
      sched[0] = p.shared_q ? -1 : 0;
      sched[1] = p.shared_q ? n * p.heads * ((query_tiles_of(p, 0) + 1) >> 1) : p.num_units;
    }
    __syncthreads();
    return;
  }
  int* s_cost = s_pre;  // key tiles per sequence, before s_pre holds the prefix
  for (int i = threadIdx.x; i < n; i += blockDim.x)
    s_cost[i] = (__ldg(p.cu_k + i + 1) - __ldg(p.cu_k + i) + kTileN - 1) / kTileN;
  {
    int* m = sched + kSchedMeta;
    const int nq = p.shared_q ? 1 : n;
    for (int i = threadIdx.x; i <= nq; i += blockDim.x) {
      m[i] = __ldg(p.cu_q + i);
      m[(kMaxSortSeqs + 1) + i] = __ldg(p.so_q + i);
    }
    for (int i = threadIdx.x; i <= n; i += blockDim.x) {
      m[2 * (kMaxSortSeqs + 1) + i] = __ldg(p.cu_k + i);
      m[3 * (kMaxSortSeqs + 1) + i] = __ldg(p.so_k + i);
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int ci = s_cost[i];
    int rank = 0;
    for (int j = 0; j < n; ++j) {
      const int cj = s_cost[j];
      rank += (cj > ci || (cj == ci && j < i)) ? 1 : 0;
    }
    s_order[rank] = i;
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    int carry = 0;
    for (int base = 0; base < n; base += 32) {
      const int r = base + static_cast<int>(threadIdx.x);
      int v = 0;
      if (r < n) {  // query tiles of the sequence, from the shared-memory copy of scale_off_q
        const int* soq = sched + kSchedMeta + (kMaxSortSeqs + 1);
        const int qs = p.shared_q ? 0 : s_order[r];
        v = p.heads * ((soq[qs + 1] - soq[qs] + 1) >> 1);
      }
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int o = __shfl_up_sync(0xFFFFFFFFu, v, d);
        if (threadIdx.x >= static_cast<unsigned>(d)) v += o;
      }
      if (r < n) s_pre[r + 1] = carry + v;
      carry += __shfl_sync(0xFFFFFFFFu, v, 31);
    }
    if (threadIdx.x == 0) {
      s_pre[0] = 0;
      sched[0] = n;
      const int grid = static_cast<int>(gridDim.x);
      const int r = carry % grid;
      const int split = (r > 0 && 2 * r <= grid) ? r : 0;
      sched[kSchedSplit] = carry - split;
      sched[1] = carry + split;
    }
  }
  __syncthreads();
}

__device__ __forceinline__ PairUnit pair_unit(const AttnParams& p, const int* sched, int w) {
  PairUnit u;
  const int n = sched[0];
  if (n > 0) {
    // Everything from shared memory: the order, its prefix and the metadata copies.
    const int* order = sched + 2;
    const int* pre = sched + 2 + kMaxSortSeqs;
    const int* cuq = sched + kSchedMeta;
    const int* soq = cuq + (kMaxSortSeqs + 1);
    const int* cuk = soq + (kMaxSortSeqs + 1);
    const int* sok = cuk + (kMaxSortSeqs + 1);
    // Units of the split tail: single tiles, two per pair of the order.
    const int keep = sched[kSchedSplit];
    const int half = w >= keep ? ((w - keep) & 1) : -1;
    const int wp = w >= keep ? keep + ((w - keep) >> 1) : w;
    const int r = find_prefix_smem(pre, n, wp);
    u.seq = order[r];
    const int local = wp - pre[r];
    const int qseq = p.shared_q ? 0 : u.seq;
    const int nt = soq[qseq + 1] - soq[qseq];
    const int np = (nt + 1) >> 1;
    u.h = local / np;
    const int pair = local - u.h * np;
    u.qtile0 = 2 * pair + (half > 0 ? 1 : 0);
    u.sbq = soq[qseq] + u.qtile0;
    u.has_q1 = (half < 0 && 2 * pair + 1 < nt) ? 1 : 0;
    const int cq0 = cuq[qseq];
    u.q_row0 = cq0 + u.qtile0 * kTileM;
    u.q_len = cuq[qseq + 1] - cq0;
    u.o_row0 = p.shared_q ? u.seq * u.q_len + u.qtile0 * kTileM : u.q_row0;
    u.k_row0 = cuk[u.seq];
    u.k_len = cuk[u.seq + 1] - u.k_row0;
    u.nkv = u.qtile0 < nt ? (u.k_len + kTileN - 1) / kTileN : -1;
    u.sbk = sok[u.seq];
    return u;
  }
  if (n < 0) {  // shared query set, plain order
    const int nt = query_tiles_of(p, 0);
    const int np = (nt + 1) >> 1;
    u.seq = w / (p.heads * np);
    const int local = w - u.seq * (p.heads * np);
    u.h = local / np;
    const int pair = local - u.h * np;
    u.qtile0 = 2 * pair;
    u.sbq = __ldg(p.so_q) + 2 * pair;
    u.has_q1 = (2 * pair + 1 < nt) ? 1 : 0;
  } else {
    u.h = w / p.total_q_tiles;
    const int g = w - u.h * p.total_q_tiles;
    u.seq = find_prefix(p.so_q, p.num_seqs, g);
    u.qtile0 = g - __ldg(p.so_q + u.seq);
    u.sbq = g;
    u.has_q1 = 0;
  }
  const int qseq = p.shared_q ? 0 : u.seq;
  const int cq0 = __ldg(p.cu_q + qseq);
  u.q_row0 = cq0 + u.qtile0 * kTileM;
  u.q_len = __ldg(p.cu_q + qseq + 1) - cq0;
  u.o_row0 = p.shared_q ? u.seq * u.q_len + u.qtile0 * kTileM : u.q_row0;
  u.k_row0 = __ldg(p.cu_k + u.seq);
  u.k_len = __ldg(p.cu_k + u.seq + 1) - u.k_row0;
  u.nkv = (u.k_len + kTileN - 1) / kTileN;
  u.sbk = __ldg(p.so_k + u.seq);
  return u;
}

__device__ __forceinline__ PairUnit warp_uniform(const PairUnit& u) {
  PairUnit r;
  r.h = lpfa::warp_uniform(u.h);
  r.seq = lpfa::warp_uniform(u.seq);
  r.qtile0 = lpfa::warp_uniform(u.qtile0);
  r.q_row0 = lpfa::warp_uniform(u.q_row0);
  r.o_row0 = lpfa::warp_uniform(u.o_row0);
  r.q_len = lpfa::warp_uniform(u.q_len);
  r.k_row0 = lpfa::warp_uniform(u.k_row0);
  r.k_len = lpfa::warp_uniform(u.k_len);
  r.nkv = lpfa::warp_uniform(u.nkv);
  r.sbq = lpfa::warp_uniform(u.sbq);
  r.sbk = lpfa::warp_uniform(u.sbk);
  r.has_q1 = lpfa::warp_uniform(u.has_q1);
  return r;
}

// Tuning switches (compile time).
// LPFA_PP_SUSPEND_NS: > 0 lets the producer and MMA-issuer warps sleep in their barrier waits
//   (suspend hint in ns) instead of spinning, leaving issue slots to the softmax warps that share
//   their SM sub-partitions.
// LPFA_PP_MAX2: the row maximum as a tree of two-input maxima instead of three-input ones.
// LPFA_PP_POLY: how many of every 8 four-key groups take their exponentials from the cubic on the
//   FMA pipe instead of the MUFU.
#ifndef LPFA_PP_SUSPEND_NS
#define LPFA_PP_SUSPEND_NS 2000
#endif
#ifndef LPFA_PP_MAX2
#define LPFA_PP_MAX2 1
#endif
#ifndef LPFA_PP_POLY
#define LPFA_PP_POLY 0
#endif
// LPFA_PP_SFREE_SPIN: the QK issuer spins (no suspend) on the S buffer's release.
#ifndef LPFA_PP_SFREE_SPIN
#define LPFA_PP_SFREE_SPIN 0
#endif

// Bounded barrier wait by a whole warp (every lane polls; warp-uniform result), sleeping between
// polls when `suspend` is set. (Having one lane poll and the others wait for it measured far
// slower.)
__device__ __forceinline__ bool wait_warp(uint64_t* bar, uint32_t parity, const volatile int* abort, bool suspend) {
  if (suspend && LPFA_PP_SUSPEND_NS > 0)
    return __all_sync(0xFFFFFFFFu, mbar_wait_suspend(bar, parity, abort, LPFA_PP_SUSPEND_NS));
  return mbar_wait_warp(bar, parity, abort);
}

// Barrier wait of the producer and issuer warps (they may sleep while waiting).
__device__ __forceinline__ bool wait_role(uint64_t* bar, uint32_t parity, const volatile int* abort) {
  return wait_warp(bar, parity, abort, true);
}

// Row maximum of the 128 S values of this thread's row.
__device__ __forceinline__ float row_max(const float2 (&s)[64]) {
#if LPFA_PP_MAX2
  float a[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) a[k] = fmaxf(s[k].x, s[k].y);
#pragma unroll
  for (int i = 8; i < 64; ++i) a[i & 7] = fmaxf(a[i & 7], fmaxf(s[i].x, s[i].y));
  return fmaxf(fmaxf(fmaxf(a[0], a[1]), fmaxf(a[2], a[3])), fmaxf(fmaxf(a[4], a[5]), fmaxf(a[6], a[7])));
#else
  return rowmax128(s);
#endif
}

// p = 2^(s c + nb) for the row's 128 keys and their E4M3 codes, in one pass: each group of four
// keys gets its scale FMAs, four exponentials, its share of the sum and its conversion together, so
// the FMA-pipe and conversion work hides under the MUFU time of the neighbouring groups instead
// of running as separate passes while the MUFU idles. Masked keys hold s = -inf and give exactly
// 0. pk receives the codes, four keys per word in key order; returns the sum of the unrounded p.
// (One call site per kernel: the loop is fully unrolled and inlined.)
__device__ __forceinline__ float exp_row_e4m3(const float2 (&s)[64], float c, float nb, uint32_t (&pk)[32]) {
  const float2 c2 = make_float2(c, c), nb2 = make_float2(nb, nb);
  float2 acc[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) acc[k] = make_float2(0.0f, 0.0f);
#pragma unroll
  for (int w = 0; w < 32; ++w) {
    const bool poly = (w & 7) < LPFA_PP_POLY;
    const float2 xa = __ffma2_rn(s[2 * w], c2, nb2), xb = __ffma2_rn(s[2 * w + 1], c2, nb2);
    const float2 a = poly ? exp2_poly2(xa) : exp2_mufu2(xa);
    const float2 b = poly ? exp2_poly2(xb) : exp2_mufu2(xb);
    acc[w & 3] = __fadd2_rn(acc[w & 3], __fadd2_rn(a, b));
    pk[w] = static_cast<uint32_t>(cvt_e4m3x2(a.x, a.y)) | (static_cast<uint32_t>(cvt_e4m3x2(b.x, b.y)) << 16);
  }
  const float2 t = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
  return t.x + t.y;
}

// bf16 P in shared memory: p = 2^(s c + nb) for the row's 128 keys, rounded to BF16 and written,
// eight keys at a time from inside the loop, as the row's 256 bytes of a K-major operand tile with
// the 128-byte swizzle (keys [64a, 64a + 64) in atom a; 16-byte chunk c of row r at byte
// (c ^ (r & 7)) * 16 of the row), so the rounded P never has to be held in registers. prow: this
// row's first byte in atom 0 (tile + r * 128). *lsum receives the sum of the unrounded p, *lrsum
// that of the BF16 values written (the weights the PV product uses). Masked keys (s = -inf) give 0.
__device__ __forceinline__ void exp_row_bf16_store(const float2 (&s)[64], float c, float nb, uint8_t* prow,
                                                   uint32_t rsw, float* lsum, float* lrsum) {
  const float2 c2 = make_float2(c, c), nb2 = make_float2(nb, nb);
  float2 acc[2] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)};
  float2 racc[2] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)};
#pragma unroll
  for (int ch = 0; ch < 16; ++ch) {  // keys [8 ch, 8 ch + 8)
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 x = exp2_mufu2(__ffma2_rn(s[4 * ch + k], c2, nb2));
      acc[k & 1] = __fadd2_rn(acc[k & 1], x);
      w[k] = cvt_bf16x2(x.x, x.y);
      racc[k & 1] = __fadd2_rn(racc[k & 1], make_float2(__uint_as_float(w[k] << 16), __uint_as_float(w[k] & 0xFFFF0000u)));
    }
    const uint32_t atom = static_cast<uint32_t>(ch) >> 3, cc = static_cast<uint32_t>(ch) & 7u;
    *reinterpret_cast<uint4*>(prow + atom * kBfAtomBytes + ((cc ^ rsw) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
  }
  const float2 t = __fadd2_rn(acc[0], acc[1]), tr = __fadd2_rn(racc[0], racc[1]);
  *lsum = t.x + t.y;
  *lrsum = tr.x + tr.y;
}

// bf16 P in TMEM: p = 2^(s c + nb) in place for the row's 128 keys (one pass of scale FMAs, exponentials
// and sums, as exp_row_e4m3); masked keys (s = -inf) give 0. Returns the sum of the unrounded p.
__device__ __forceinline__ float exp_row_inplace(float2 (&s)[64], float c, float nb) {
  const float2 c2 = make_float2(c, c), nb2 = make_float2(nb, nb);
  float2 acc[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) acc[k] = make_float2(0.0f, 0.0f);
#pragma unroll
  for (int i = 0; i < 64; ++i) {
    s[i] = exp2_mufu2(__ffma2_rn(s[i], c2, nb2));
    acc[i & 3] = __fadd2_rn(acc[i & 3], s[i]);
  }
  const float2 t = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
  return t.x + t.y;
}

// Row reference of the online softmax in the fp8 PV mode: P = E4M3(2^(kBias - m) 2^t) with the
// integer reference m trailing the row's running ceiling by at most kLag binades, so P <= 2^8 <
// 448. With three binades of lag a row's reference (and with it O, by an exact power of two)
// moves about ten times less often than with two on unit-variance logits, once past the first tiles.
constexpr float kLagP8 = 3.0f;
constexpr float kBiasP8 = 5.0f;

template <int kPv, bool kPerUnitDescale>
__global__ void __launch_bounds__(kAttnThreads, 1)
attn_fwd_pp_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                   const __grid_constant__ CUtensorMap tmap_v, const AttnParams p) {
  using L = Smem<kPv>;
  constexpr bool kMx = kPv == kPvMx;        // block-scaled MXFP8 PV: P and V scaled per 32 keys
  constexpr bool kBf = L::kBf;              // bf16 P, BF16 V in shared memory
  constexpr bool kPSm = L::kPS_;            // bf16 P in shared memory (else in one TMEM slot)
  constexpr bool kVIn = L::kVIn;            // BF16 V input (TMA straight into the operand layout)
  constexpr bool kConv = kPv == kPvBf16Mx;  // MXFP8 V converted to BF16 by warps 12..15
  constexpr bool kEpi = !kConv && LPFA_PP_EPI_WG;  // warps 12..15 write O and LSE (else the softmax warps do)
  // bf16 P: the softmax warps decode the next unit one unit ahead (measured +1.5-2.5 % on
  // 16-key-tile units; with 8-bit P the registers it holds through the unit cost 2-5 %).
  constexpr bool kNextUnit = kBf;
  constexpr int kQS = L::kQS, kKS = L::kKS;
  // Ring depths as divisors: a ring a mode does not use has depth 0 in L; its code is never reached.
  constexpr int kVS = L::kVS > 0 ? L::kVS : 1, kVBS = L::kVBS > 0 ? L::kVBS : 1;
  constexpr uint32_t kNSlots = kBf ? kPSlotsBf : kPSlots;
  // PV completions go to PVDone[n % kNBarsPV]. With one P slot they alternate between two barriers:
  // a warpgroup waiting for PV n - 1 knows PV n - 3 complete and PV n + 1 impossible yet, so the
  // phase it asks for is never two completions away (on a single barrier it could be).
  constexpr uint32_t kNBarsPV = kNSlots == 1 ? 2 : kNSlots;
  constexpr uint32_t kSfaBase = kBf ? kColSFABf : kColSFA8;  // early-copied scale atoms (fp8, bf16 PV)
  constexpr uint32_t kSfbBase = kBf ? kColSFBBf : kColSFB8;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::bars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::misc + 16);
  int* sched_w = reinterpret_cast<int*>(smem + L::sched);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kQS; ++i) { mbar_init(&bars[kBarQFull + i], 1); mbar_init(&bars[kBarQEmpty + i], 1); }
    for (int i = 0; i < kKS; ++i) { mbar_init(&bars[kBarKFull + i], 1); mbar_init(&bars[kBarKEmpty + i], 1); }
    for (int i = 0; i < L::kVS; ++i) {
      mbar_init(&bars[kBarVFull + i], 1);
      mbar_init(&bars[kBarVEmpty + i], kConv ? 4 : 1);  // the 4 converter warps, or an MMA commit
    }
    for (int i = 0; i < L::kVBS; ++i) {
      mbar_init(&bars[kBarVbfFull + i], kVIn ? 1 : 4);  // the V producer's TMA, or the 4 converter warps
      mbar_init(&bars[kBarVbfEmpty + i], 1);
    }
    mbar_init(&bars[kBarSFree], 4);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars[kBarSFull + i], 1);
      mbar_init(&bars[kBarOFull + i], 1);
      mbar_init(&bars[kBarOEmpty + i], 4);
    }
    for (uint32_t i = 0; i < kNSlots; ++i) {
      // PReady counts the 4 warps of the storing warpgroup; an arrival for the slot's next P
      // needs the PV of this one complete, so the phases of one slot cannot mix.
      mbar_init(&bars[kBarPReady + i], 4);
    }
    for (uint32_t i = 0; i < kNBarsPV; ++i) mbar_init(&bars[kBarPVDone + i], 1);
    mbar_init(&bars[kBarDrain], 1);
    mbar_init(&bars[kBarDrainPV], 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars[kBarStatsFull + i], 4);
      mbar_init(&bars[kBarStatsFree + i], 4);
    }
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmap_q);
    prefetch_tmap(&tmap_k);
    prefetch_tmap(&tmap_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  build_pair_order(p, sched_w);
  const int* sched = sched_w;
  const int num_units = sched[1];
  // One CTA per SM owns all 512 columns, so the allocation starts at lane 0, column 0; using the
  // constant keeps every TMEM operand a compile-time or warp-uniform value.
  constexpr uint32_t tmem = 0;
  const bool tmem_ok = *tmem_slot == tmem;
  if (!tmem_ok && threadIdx.x == 0) record_failure(abort_flag, kPSiteTmem);

  const int G = gridDim.x;

  if (!tmem_ok) {
    // nothing issued; fall through to the teardown
  } else if (warp < 4) {
    setmaxnreg_dec<kOtherRegs>();
    const uint32_t leader = lane == 0 ? 1u : 0u;
    if (warp == 0) {
      // ---------------------------------------------------------------- Q/K producer
      uint32_t qc = 0, kc = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < num_units && ok; w += G) {
        const PairUnit ui = warp_uniform(pair_unit(p, sched, w));
        if (ui.nkv <= 0) continue;  // no keys (the softmax warps write the empty-sum result), or no tile
        const uint32_t qs = qc % kQS, qph = (qc / kQS) & 1;
        if (!wait_role(&bars[kBarQEmpty + qs], qph ^ 1, abort_flag)) { record_failure(abort_flag, kPSiteProducerQ); ok = false; break; }
        mbar_arrive_expect_tx(&bars[kBarQFull + qs], (ui.has_q1 ? 2u : 1u) * (kTileBytes + kAtomBytes), leader);
        for (int i = 0; i <= ui.has_q1; ++i) {
          tma_load_3d(smem + L::q + (qs * 2 + i) * kTileBytes, &tmap_q, &bars[kBarQFull + qs], 0, ui.h,
                      ui.q_row0 + i * kTileM, leader);
          bulk_load(smem + L::q_sf + (qs * 2 + i) * kAtomBytes,
                    p.q_sf + (static_cast<int64_t>(ui.sbq + i) * p.heads + ui.h) * kAtomBytes, kAtomBytes,
                    &bars[kBarQFull + qs], leader);
        }
        ++qc;
        if (kQS == 1 && w + G < num_units) {
          // With one Q stage the next unit's tiles can only be loaded once this unit's last QK
          // has run; bring them into L2 now so that load is an L2 hit.
          const PairUnit un = warp_uniform(pair_unit(p, sched, w + G));
          if (un.nkv > 0)
            for (int i = 0; i <= un.has_q1; ++i) tma_prefetch_3d(&tmap_q, 0, un.h, un.q_row0 + i * kTileM, leader);
        }
        for (int j = 0; j < ui.nkv; ++j) {
          const uint32_t s = kc % kKS, ph = (kc / kKS) & 1;
          if (!wait_role(&bars[kBarKEmpty + s], ph ^ 1, abort_flag)) { record_failure(abort_flag, kPSiteProducerK); ok = false; break; }
          mbar_arrive_expect_tx(&bars[kBarKFull + s], kTileBytes + kAtomBytes, leader);
          tma_load_3d(smem + L::k + s * kTileBytes, &tmap_k, &bars[kBarKFull + s], 0, ui.h, ui.k_row0 + j * kTileN,
                      leader);
          bulk_load(smem + L::k_sf + s * kAtomBytes,
                    p.k_sf + (static_cast<int64_t>(ui.sbk + j) * p.heads + ui.h) * kAtomBytes, kAtomBytes,
                    &bars[kBarKFull + s], leader);
          ++kc;
        }
      }
      // Drain: every copy issued here lands before the CTA exits (the newest fill of each stage
      // is the last one issued into it; older fills were consumed already).
      for (uint32_t i = (qc > kQS ? qc - kQS : 0); i < qc; ++i)
        if (!mbar_wait(&bars[kBarQFull + i % kQS], (i / kQS) & 1, nullptr)) record_failure(abort_flag, kPSiteDrain);
      for (uint32_t i = (kc > kKS ? kc - kKS : 0); i < kc; ++i)
        if (!mbar_wait(&bars[kBarKFull + i % kKS], (i / kKS) & 1, nullptr)) record_failure(abort_flag, kPSiteDrain);
    } else if (warp == 3 && kVIn) {
      // ---------------------------------------------------------------- V producer (BF16 V)
      // Two TMA boxes per tile (head_dim [0, 64) and [64, 128), 128 keys each, 128-byte swizzle)
      // are exactly the MN-major BF16 operand layout the PV MMA reads.
      uint32_t vc = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < num_units && ok; w += G) {
        const PairUnit ui = warp_uniform(pair_unit(p, sched, w));
        for (int j = 0; j < ui.nkv; ++j) {
          const uint32_t sb = vc % kVBS, ph = (vc / kVBS) & 1;
          if (!wait_role(&bars[kBarVbfEmpty + sb], ph ^ 1, abort_flag)) { record_failure(abort_flag, kPSiteProducerV); ok = false; break; }
          mbar_arrive_expect_tx(&bars[kBarVbfFull + sb], kBfTileBytes, leader);
#pragma unroll
          for (int a = 0; a < 2; ++a)
            tma_load_3d(smem + L::vbf + sb * kBfTileBytes + a * kBfAtomBytes, &tmap_v, &bars[kBarVbfFull + sb], a * 64,
                        ui.h, ui.k_row0 + j * kTileN, leader);
          ++vc;
        }
      }
      for (uint32_t i = (vc > kVBS ? vc - kVBS : 0); i < vc; ++i)
        if (!mbar_wait(&bars[kBarVbfFull + i % kVBS], (i / kVBS) & 1, nullptr)) record_failure(abort_flag, kPSiteDrain);
    } else if (warp == 3) {
      // ---------------------------------------------------------------- V producer (8-bit V)
      uint32_t vc = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < num_units && ok; w += G) {
        const PairUnit ui = warp_uniform(pair_unit(p, sched, w));
        for (int j = 0; j < ui.nkv; ++j) {
          const uint32_t s = vc % kVS, ph = (vc / kVS) & 1;
          if (!wait_role(&bars[kBarVEmpty + s], ph ^ 1, abort_flag)) { record_failure(abort_flag, kPSiteProducerV); ok = false; break; }
          mbar_arrive_expect_tx(&bars[kBarVFull + s], kTileBytes + (L::kVsf ? kAtomBytes : 0u), leader);
          tma_load_3d(smem + L::v + s * kTileBytes, &tmap_v, &bars[kBarVFull + s], 0, ui.h, ui.k_row0 + j * kTileN,
                      leader);
          if (L::kVsf)
            bulk_load(smem + L::v_sf + s * kAtomBytes,
                      p.v_sf + (static_cast<int64_t>(ui.sbk + j) * p.heads + ui.h) * kAtomBytes, kAtomBytes,
                      &bars[kBarVFull + s], leader);
          ++vc;
        }
      }
      for (uint32_t i = (vc > kVS ? vc - kVS : 0); i < vc; ++i)
        if (!mbar_wait(&bars[kBarVFull + i % kVS], (i / kVS) & 1, nullptr)) record_failure(abort_flag, kPSiteDrain);
    } else if (warp == 1) {
      // ---------------------------------------------------------------- QK issuer
      // The S buffer is used in the order (unit, key tile j, query tile i); each use waits until
      // the previous one has been read out (SFree), which also guarantees that every earlier
      // QK, and with it every earlier read of a scale-factor slot, has completed.
      const uint32_t sb = static_cast<uint32_t>(lpfa::warp_uniform(static_cast<int>(smem_u32(smem))));
      const uint64_t dq0 = umma_desc(sb + L::q, 16, 1024, kLayoutSw128);
      const uint64_t dk0 = umma_desc(sb + L::k, 16, 1024, kLayoutSw128);
      const uint64_t dqsf0 = umma_desc(sb + L::q_sf, 0, 128, kLayoutNone);
      const uint64_t dksf0 = umma_desc(sb + L::k_sf, 0, 128, kLayoutNone);
      uint32_t u = 0, kc = 0, uses = 0;
      bool ok = true;
      if (p.debug_stall > 0) {
        // Test hook: wait for a phase of the drain barrier that nothing completes before the
        // drains below, so the wait runs out and the failure path is exercised.
        if (!wait_role(&bars[kBarDrain], 0, abort_flag)) { record_failure(abort_flag, kPSiteDebugStall); ok = false; }
      }
      // The sign of the logit scale goes into the MMA (negated A); the softmax uses |scale|. The
      // descales are global loads: each unit's are issued one unit ahead, so that their latency is
      // not between the last QK of one unit and the first of the next.
      float qd_next = 1.0f, kd_next = 1.0f;
      if (static_cast<int>(blockIdx.x) < num_units) {
        const PairUnit u0 = warp_uniform(pair_unit(p, sched, blockIdx.x));
        qd_next = descale_value(p.q_descale, u0.seq, u0.h);
        kd_next = descale_value(p.k_descale, u0.seq, u0.h);
      }
      for (int w = blockIdx.x; w < num_units && ok; w += G) {
        const PairUnit ui = warp_uniform(pair_unit(p, sched, w));
        const float qd = qd_next, kd = kd_next;
        if (w + G < num_units) {
          const PairUnit un = warp_uniform(pair_unit(p, sched, w + G));
          qd_next = descale_value(p.q_descale, un.seq, un.h);
          kd_next = descale_value(p.k_descale, un.seq, un.h);
        }
        if (ui.nkv <= 0) continue;
        const int negate = (qd * kd) < 0.0f ? 1 : 0;
        uint32_t idq[4];
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) idq[kk] = idesc_qk(kk, negate);
        const uint32_t qs = u % kQS;
        if (!wait_role(&bars[kBarQFull + qs], (u / kQS) & 1, abort_flag)) { record_failure(abort_flag, kPSiteMmaQ); ok = false; break; }
        // Early-copied Q atoms (fp8 and bf16 PV): both tiles' atoms into this unit stage's slots.
        // With two stages their last reader, the unit two back, completed before the first QK of
        // the previous unit could write S, so they are copied now; with one stage (bf16 PV) the
        // last reader is the previous unit, and the copy waits for the unit's first S release.
        auto copy_q_atoms = [&]() {
          tc_fence_after();
          for (int i = 0; i <= ui.has_q1; ++i)
            tmem_cp_32x128b_x4(tmem + kSfaBase + qs * 8 + i * 4, dqsf0 + ((qs * 2 + i) * kAtomBytes >> 4), leader);
        };
        if (!kMx && kQS > 1) copy_q_atoms();
        // K tile kc is waited for, and (early-copy modes) its atom copied into slot kc & 1, right
        // after the previous tile's last QK has been issued, so that neither sits between the next
        // SFree and the next QK. The slot's last reader, a QK of tile kc - 2, completed before the S
        // that the last SFree released was written.
        auto prepare_k = [&]() -> bool {
          if (!wait_role(&bars[kBarKFull + kc % kKS], (kc / kKS) & 1, abort_flag)) return false;
          if (!kMx) {
            tc_fence_after();
            tmem_cp_32x128b_x4(tmem + kSfbBase + (kc & 1) * 4, dksf0 + ((kc % kKS) * kAtomBytes >> 4), leader);
          }
          return true;
        };
        if (!prepare_k()) { record_failure(abort_flag, kPSiteMmaK); ok = false; break; }
        for (int j = 0; j < ui.nkv && ok; ++j) {
          const uint32_t s = kc % kKS;
          const uint64_t bdesc = dk0 + (s * kTileBytes >> 4);
          const uint32_t sfb = tmem + (kMx ? kColSFB : kSfbBase + (kc & 1) * 4);
          for (int i = 0; i <= ui.has_q1; ++i) {
            if (uses > 0) {
#if LPFA_PP_SFREE_SPIN
              if (!mbar_wait_warp(&bars[kBarSFree], (uses - 1) & 1, abort_flag)) { record_failure(abort_flag, kPSiteMmaS); ok = false; break; }
#else
              if (!wait_role(&bars[kBarSFree], (uses - 1) & 1, abort_flag)) { record_failure(abort_flag, kPSiteMmaS); ok = false; break; }
#endif
            }
            tc_fence_after();
            if (!kMx && kQS == 1 && j == 0 && i == 0) copy_q_atoms();
            const uint32_t sfa = tmem + (kMx ? kColSFA : kSfaBase + qs * 8 + i * 4);
            if (kMx) {
              // Scale atoms into their single TMEM slots, in order with the MMAs below. The QK that
              // last read them wrote the previous S, which its warpgroup has read out (SFree), so
              // it has completed.
              tmem_cp_32x128b_x4(sfa, dqsf0 + ((qs * 2 + i) * kAtomBytes >> 4), leader);
              if (i == 0) tmem_cp_32x128b_x4(sfb, dksf0 + (s * kAtomBytes >> 4), leader);
            }
            const uint64_t adesc = dq0 + ((qs * 2 + i) * kTileBytes >> 4);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {  // K = 32 bytes per MMA, scale byte kk
              const uint32_t byte_sel = static_cast<uint32_t>(kk) << 30;
              mma_mxf8f6f4_ss(tmem + kColS, adesc + kk * 2, bdesc + kk * 2, idq[kk], sfa | byte_sel, sfb | byte_sel,
                              kk > 0 ? 1u : 0u, leader);
            }
            mma_commit(&bars[kBarSFull + i], leader);
            ++uses;
          }
          if (!ok) break;
          mma_commit(&bars[kBarKEmpty + s], leader);
          if (j == ui.nkv - 1) mma_commit(&bars[kBarQEmpty + qs], leader);
          ++kc;
          if (j + 1 < ui.nkv && !prepare_k()) { record_failure(abort_flag, kPSiteMmaK); ok = false; break; }
        }
        ++u;
      }
      mma_commit(&bars[kBarDrain], leader);
      if (!mbar_wait(&bars[kBarDrain], 0, nullptr)) record_failure(abort_flag, kPSiteDrain);
    } else {
      // ---------------------------------------------------------------- PV issuer (warp 2)
      const uint32_t sb = static_cast<uint32_t>(lpfa::warp_uniform(static_cast<int>(smem_u32(smem))));
      const uint64_t dv0 = umma_desc(sb + L::v, kTileBytes, 1024, kLayoutSw128);       // 8-bit V, MN-major
      const uint64_t dvb0 = umma_desc(sb + L::vbf, kBfAtomBytes, 1024, kLayoutSw128);  // BF16 V, MN-major
      const uint64_t dpb0 = umma_desc(sb + L::pbf, 16, 1024, kLayoutSw128);            // bf16 P, K-major
      const uint64_t dpsf0 = umma_desc(sb + L::p_sf, 0, 128, kLayoutNone);
      const uint64_t dvsf0 = umma_desc(sb + L::v_sf, 0, 128, kLayoutNone);
      uint32_t vc = 0;          // V tiles
      uint32_t n = 0;           // P tiles, in the order the PVs consume them
      uint32_t uc[2] = {0, 0};  // units per warpgroup
      bool ok = true;
      for (int w = blockIdx.x; w < num_units && ok; w += G) {
        const PairUnit ui = warp_uniform(pair_unit(p, sched, w));
        if (ui.nkv <= 0) continue;
        for (int j = 0; j < ui.nkv && ok; ++j) {
          const uint32_t vs = kBf ? vc % kVBS : vc % kVS;
          // V first: it is loaded well ahead, so this wait is off the path from P to PV.
          const bool vok = kBf ? wait_role(&bars[kBarVbfFull + vs], (vc / kVBS) & 1, abort_flag)
                               : wait_role(&bars[kBarVFull + vs], (vc / kVS) & 1, abort_flag);
          if (!vok) { record_failure(abort_flag, kPSiteMmaV); ok = false; break; }
          for (int i = 0; i <= ui.has_q1; ++i) {
            const uint32_t ps = n % kNSlots;
            if (!wait_role(&bars[kBarPReady + ps], (n / kNSlots) & 1, abort_flag)) { record_failure(abort_flag, kPSiteMmaP); ok = false; break; }
            if (j == 0 && !wait_role(&bars[kBarOEmpty + i], (uc[i] & 1) ^ 1, abort_flag)) { record_failure(abort_flag, kPSiteMmaO); ok = false; break; }
            tc_fence_after();
            const uint32_t o_col = tmem + kColO + i * 128;
            if (kBf && kPSm) {
              // BF16: P (K-major) and V (MN-major) from shared memory, K = 16 keys per MMA.
              const uint64_t adesc = dpb0 + (ps * kBfTileBytes >> 4);
              const uint64_t bdesc = dvb0 + (vs * kBfTileBytes >> 4);
#pragma unroll
              for (int kk = 0; kk < 8; ++kk)
                mma_f16_ss(o_col, adesc + (kk >> 2) * (kBfAtomBytes >> 4) + (kk & 3) * 2, bdesc + kk * 128,
                           kIdescPV16, (j > 0 || kk > 0) ? 1u : 0u, leader);
            } else if (kBf) {
              // BF16: P from its TMEM slot (2 keys per column), V (MN-major) from shared memory.
              const uint64_t bdesc = dvb0 + (vs * kBfTileBytes >> 4);
#pragma unroll
              for (int kk = 0; kk < 8; ++kk)  // keys [16kk, 16kk + 16): 8 columns of 2 BF16 each
                mma_f16_ts(o_col, tmem + kColP + kk * 8, bdesc + kk * 128, kIdescPV16, (j > 0 || kk > 0) ? 1u : 0u,
                           leader);
            } else if (kMx) {
              // Scale atoms into TMEM, in order with the MMAs below: V's once per V tile into slot
              // vc % 3, P's from the softmax's shared-memory atom of this P slot into the matching
              // TMEM slot. Before storing this P the softmax waited for the PV three P tiles
              // back, so every PV that read either slot earlier has completed.
              const uint32_t p_col = tmem + kColP + ps * 32;
              const uint64_t bdesc = dv0 + (vs * kTileBytes >> 4);
              const uint32_t sfv = tmem + kColSFV + (vc % 3) * 4;
              const uint32_t sfp = tmem + kColSFP + ps * 4;
              if (i == 0) tmem_cp_32x128b_x4(sfv, dvsf0 + (vs * kAtomBytes >> 4), leader);
              tmem_cp_32x128b_x4(sfp, dpsf0 + (ps * kAtomBytes >> 4), leader);
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {  // keys [32kk, 32kk + 32), scale byte kk
                const uint32_t byte_sel = static_cast<uint32_t>(kk) << 30;
                mma_mxf8f6f4_ts(o_col, p_col + kk * 8, bdesc + kk * 256, idesc_pv_mx(kk), sfp | byte_sel,
                                sfv | byte_sel, (j > 0 || kk > 0) ? 1u : 0u, leader);
              }
            } else {
              const uint32_t p_col = tmem + kColP + ps * 32;
              const uint64_t bdesc = dv0 + (vs * kTileBytes >> 4);
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)  // keys [32kk, 32kk + 32): 8 columns of 4 E4M3 each
                mma_f8f6f4_ts(o_col, p_col + kk * 8, bdesc + kk * 256, kIdescPV8, (j > 0 || kk > 0) ? 1u : 0u, leader);
            }
            mma_commit(&bars[kBarPVDone + n % kNBarsPV], leader);
            ++n;
          }
          if (!ok) break;
          mma_commit(kBf ? &bars[kBarVbfEmpty + vs] : &bars[kBarVEmpty + vs], leader);
          ++vc;
        }
        if (!ok) break;
        for (int i = 0; i <= ui.has_q1; ++i) {
          mma_commit(&bars[kBarOFull + i], leader);  // every PV_i of this unit is complete
          ++uc[i];
        }
      }
      mma_commit(&bars[kBarDrainPV], leader);
      if (!mbar_wait(&bars[kBarDrainPV], 0, nullptr)) record_failure(abort_flag, kPSiteDrain);
    }
  } else if (warp < 12) {
    setmaxnreg_inc<kSoftmaxRegs>();
    // ------------------------------------------------------------------ softmax warpgroups
    // (Block-scaled and bf16 P have no E4M3 range limit to respect: they take a lag of 8 binades.)
    constexpr float kLag = kPv == kPvFp8 ? kLagP8 : kLagWide;
    constexpr float kBias = kPv == kPvFp8 ? kBiasP8 : kBiasWide;
    uint32_t* p_sf_words = reinterpret_cast<uint32_t*>(smem + L::p_sf);
    const int grp = (warp - 4) >> 2;                 // query tile of the unit this warpgroup owns
    const int quarter = warp & 3;                    // TMEM lane quarter of this warp
    const int row = quarter * 32 + lane;             // query row within the tile
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const float cscale_all = kPerUnitDescale ? 0.0f
                                             : fabsf((descale_value(p.q_descale, 0, 0) *
                                                      descale_value(p.k_descale, 0, 0)) * kLog2eRsqrtD);
    uint32_t sc = 0, ucnt = 0;  // S tiles read, units finished
    uint32_t nbase = 0;         // P tiles of all earlier units, in the order the PVs consume them
    float2* stats = reinterpret_cast<float2*>(smem + L::stats);
    bool ok = true;
    PairUnit ui_next;
    if (kNextUnit && static_cast<int>(blockIdx.x) < num_units) ui_next = pair_unit(p, sched, blockIdx.x);
    for (int w = blockIdx.x; w < num_units && ok; w += G) {
      const PairUnit ui = kNextUnit ? ui_next : pair_unit(p, sched, w);
      if (kNextUnit && w + G < num_units) ui_next = pair_unit(p, sched, w + G);
      const uint32_t np = 1u + static_cast<uint32_t>(ui.has_q1);  // P tiles per key tile
      const uint32_t n0 = nbase;
      nbase += static_cast<uint32_t>(max(ui.nkv, 0)) * np;
      if (grp > ui.has_q1) continue;
      const bool valid = (ui.qtile0 + grp) * kTileM + row < ui.q_len;
      const int64_t tok = ui.o_row0 + grp * kTileM + row;  // output and LSE row
      if (ui.nkv < 0) continue;  // the absent second tile of a split pair
      if (ui.nkv == 0) {
        // No keys: an empty sum, LSE = log 0 = -inf and O = 0.
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(p.out + (tok * p.heads + ui.h) * 128);
#pragma unroll
          for (int c = 0; c < 16; ++c) dst[c] = make_uint4(0u, 0u, 0u, 0u);
          p.lse[static_cast<int64_t>(ui.h) * p.tq + tok] = -INFINITY;
        }
        continue;
      }
      const float cscale = kPerUnitDescale ? fabsf((descale_value(p.q_descale, ui.seq, ui.h) *
                                                    descale_value(p.k_descale, ui.seq, ui.h)) * kLog2eRsqrtD)
                                           : cscale_all;
      const float vd = descale_value(p.v_descale, ui.seq, ui.h);  // read now, used after the last tile
      float m_r = -INFINITY;  // row reference (integer, log2 units)
      float l_r = 0.0f;       // row sum of p (times 2^kBias), relative to m_r
      float lr_r = 0.0f;      // bf16 P: the same sum over the BF16-rounded P
      for (int j = 0; j < ui.nkv; ++j) {
        if (!wait_warp(&bars[kBarSFull + grp], sc & 1, abort_flag, false)) { record_failure(abort_flag, kPSiteSoftS); ok = false; break; }
        tc_fence_after();
        float2 sv[64];
        load_row(tmem + lane_addr + kColS, sv);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[kBarSFree]);  // the S buffer may be overwritten
        ++sc;
        const int key0 = j * kTileN;
        const bool tail = key0 + kTileN > ui.k_len;
        if (tail) mask_keys(sv, key0, ui.k_len);
        // This P's slot is free once the PV kNSlots P tiles back, its previous reader, has completed.
        const uint32_t n = n0 + static_cast<uint32_t>(j) * np + static_cast<uint32_t>(grp);
        const uint32_t ps = n % kNSlots;
        auto wait_pv = [&](uint32_t m) -> bool {  // PV m complete
          if (!wait_warp(&bars[kBarPVDone + m % kNBarsPV], (m / kNBarsPV) & 1, abort_flag, false)) return false;
          tc_fence_after();
          return true;
        };
        auto wait_slot = [&]() -> bool { return n < kNSlots || wait_pv(n - kNSlots); };
        float gmax[4];  // block-scaled MXFP8 P: the 32-key group maxima of S
        float m_new;
        float psum, prsum = 0.0f;
        uint32_t mx_sfw = 0;  // block-scaled MXFP8 P: this row's four E8M0 scale bytes
        uint32_t pk[32];      // 8-bit P as E4M3 codes, four keys per word
        if (kMx) {
          // The reference moves only when the tile's ceiling exceeds it by more than the lag, so
          // the rescales are rare exact powers of two.
          const float c_t = ceilf(rowmax128_groups(sv, gmax) * cscale);
          m_new = (j == 0 || c_t > m_r + kLag) ? c_t : m_r;
          // Group g: the largest p is ex2(gmax * c + nb) (ex2 and the fma are monotonic), which
          // picks 2^e_g (RCEIL); the exponentials then run with bias nb - e_g, giving p * 2^-e_g.
          const float nb = kBias - m_new;
          float nbg[4], gsum[4];
          int eg[4];
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            eg[g] = e8m0_exponent(ex2_approx(fmaf(gmax[g], cscale, nb)), 0);
            nbg[g] = nb - static_cast<float>(eg[g]);
            mx_sfw |= static_cast<uint32_t>(eg[g] + 127) << (8 * g);
          }
          if (tail) exp_row_groups<true>(sv, cscale, nbg, key0, ui.k_len, gsum);
          else exp_row_groups<false>(sv, cscale, nbg, key0, ui.k_len, gsum);
          psum = 0.0f;
#pragma unroll
          for (int g = 0; g < 4; ++g)  // sum of the unscaled p: exact powers of two (2^-126 for an empty group)
            psum += gsum[g] * __uint_as_float(static_cast<uint32_t>(max(eg[g], -126) + 127) << 23);
#pragma unroll
          for (int c = 0; c < 32; ++c)
            pk[c] = static_cast<uint32_t>(cvt_e4m3x2(sv[2 * c].x, sv[2 * c].y)) |
                    (static_cast<uint32_t>(cvt_e4m3x2(sv[2 * c + 1].x, sv[2 * c + 1].y)) << 16);
        } else {
          // The reference moves only when the tile's ceiling exceeds it by more than the lag
          // (a unit's first tile: its own ceiling), so the rescales are rare exact powers of two.
          const float c_t = ceilf(row_max(sv) * cscale);
          m_new = (j == 0 || c_t > m_r + kLag) ? c_t : m_r;
          if (kPSm) {
            // bf16 P is written into its shared-memory slot from inside the exponential loop, so
            // the slot must be free first (normally long since: the PV two P tiles back).
            if (!wait_slot()) { record_failure(abort_flag, kPSiteSoftPV); ok = false; break; }
            exp_row_bf16_store(sv, cscale, kBias - m_new, smem + L::pbf + ps * kBfTileBytes + row * 128,
                               static_cast<uint32_t>(row & 7), &psum, &prsum);
            fence_proxy_async_smem();  // the PV MMA reads P through the async proxy
          } else if (kBf) {
            psum = exp_row_inplace(sv, cscale, kBias - m_new);
          } else {
            psum = exp_row_e4m3(sv, cscale, kBias - m_new, pk);
          }
        }
        const float m_prev = m_r;
        const float l_scale = exp2_int(m_prev - m_new);
        l_r = l_r * l_scale + psum;
        lr_r = lr_r * l_scale + prsum;  // (bf16 P in TMEM: this tile's rounded sum is added below)
        m_r = m_new;
        if (!kPSm && !wait_slot()) { record_failure(abort_flag, kPSiteSoftPV); ok = false; break; }
        if (kPSm) {
          // (stored inside the exponential loop)
        } else if (kBf) {
          // P rounded to BF16 into the slot, 32 columns (64 keys) at a time; the sum of the rounded
          // values is what O is normalised by.
          float2 racc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t pw[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              pw[c] = cvt_bf16x2(sv[32 * h + c].x, sv[32 * h + c].y);
              racc[c & 3] = __fadd2_rn(racc[c & 3], make_float2(__uint_as_float(pw[c] << 16),
                                                                __uint_as_float(pw[c] & 0xFFFF0000u)));
            }
            tmem_st32_sync(tmem + lane_addr + kColP + h * 32, pw);
          }
          const float2 rs = __fadd2_rn(__fadd2_rn(racc[0], racc[1]), __fadd2_rn(racc[2], racc[3]));
          lr_r += rs.x + rs.y;
        } else {
          if (kMx) {
            // The row's four scale bytes go to the slot's shared-memory atom (row r at
            // (r % 32) * 16 + (r / 32) * 4), read by the PV issuer's tcgen05.cp.
            p_sf_words[ps * (kAtomBytes / 4) + (row & 31) * 4 + (row >> 5)] = mx_sfw;
            fence_proxy_async_smem();
          }
          tmem_st32_sync(tmem + lane_addr + kColP + ps * 32, pk);
        }
        // O_i holds tiles up to j - 1 relative to m_prev: rescale it when the reference moved
        // (rare; never on a unit's first tile), once PV_i of tile j - 1 has completed. (That PV's
        // slot cannot have been reused yet: its next use needs this P consumed first.)
        if (j > 0 && __any_sync(0xFFFFFFFFu, m_new != m_prev)) {
          if (!wait_pv(n - np)) { record_failure(abort_flag, kPSiteSoftPV); ok = false; break; }
          const float alpha = exp2_int(m_prev - m_new);
          const float2 a2 = make_float2(alpha, alpha);
          const uint32_t o_addr = tmem + lane_addr + kColO + grp * 128;
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t ro[32];
            tmem_ld32_sync(o_addr + c * 32, ro);
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float2 o2 = __fmul2_rn(make_float2(__uint_as_float(ro[2 * e]), __uint_as_float(ro[2 * e + 1])), a2);
              ro[2 * e] = __float_as_uint(o2.x);
              ro[2 * e + 1] = __float_as_uint(o2.y);
            }
            tmem_st32_sync(o_addr + c * 32, ro);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[kBarPReady + ps]);
      }
      if (!ok) break;
      if (kEpi) {
        // Hand the row's O scale and LSE to the epilogue warpgroup and go on to the next unit. The
        // slot is free once the epilogue has read this warpgroup's previous unit's values.
        if (ucnt > 0 && !wait_warp(&bars[kBarStatsFree + grp], (ucnt - 1) & 1, abort_flag, false)) { record_failure(abort_flag, kPSiteSoftStats); ok = false; break; }
        stats[grp * kTileM + row] = make_float2(vd / (kBf ? lr_r : l_r),
                                                (m_r - kBias + lg2_approx(l_r)) * kLn2);
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[kBarStatsFull + grp]);
        ++ucnt;
        continue;
      }
      // ---------------------------------------------------------------- epilogue
      if (!wait_warp(&bars[kBarOFull + grp], ucnt & 1, abort_flag, false)) { record_failure(abort_flag, kPSiteSoftO); ok = false; break; }
      tc_fence_after();
      // O is normalised by the sum of the P values the PV product used (bf16 P: the rounded ones, so
      // a row dominated by one key gets that V row exactly); the LSE keeps the unrounded sum.
      const float oscale = vd / (kBf ? lr_r : l_r);
      uint4* dst = reinterpret_cast<uint4*>(p.out + (tok * p.heads + ui.h) * 128);
      // O_i in two halves of 64 columns; the second load releases O_i to the next unit's PV.
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        uint32_t ra[32], rb[32];
        tmem_ld64_sync(tmem + lane_addr + kColO + grp * 128 + half * 64, ra, rb);
        if (half == 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars[kBarOEmpty + grp]);
        }
        if (valid) {
          auto put = [&](const uint32_t (&r)[32], int base) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              uint4 v;
              v.x = cvt_bf16x2(__uint_as_float(r[8 * c + 0]) * oscale, __uint_as_float(r[8 * c + 1]) * oscale);
              v.y = cvt_bf16x2(__uint_as_float(r[8 * c + 2]) * oscale, __uint_as_float(r[8 * c + 3]) * oscale);
              v.z = cvt_bf16x2(__uint_as_float(r[8 * c + 4]) * oscale, __uint_as_float(r[8 * c + 5]) * oscale);
              v.w = cvt_bf16x2(__uint_as_float(r[8 * c + 6]) * oscale, __uint_as_float(r[8 * c + 7]) * oscale);
              dst[base + c] = v;
            }
          };
          put(ra, half * 8);
          put(rb, half * 8 + 4);
        }
      }
      ++ucnt;
      if (valid) p.lse[static_cast<int64_t>(ui.h) * p.tq + tok] = (m_r - kBias + lg2_approx(l_r)) * kLn2;
    }
  } else {
    setmaxnreg_dec<kOtherRegs>();
    if (kConv) {
      // ---------------------------------------------------------------- V converter (bf16 PV)
      // Thread t converts key row t of the MXFP8 V tile (E4M3 -> f16x2 exactly, times the block's
      // 2^e, -> bf16x2; exact for e >= -124) into the MN-major, 128-byte-swizzled BF16 layout.
      const int t = threadIdx.x - 12 * 32;
      const uint32_t sw = static_cast<uint32_t>(t & 7);
      uint32_t vc = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < num_units && ok; w += G) {
        const PairUnit ui = pair_unit(p, sched, w);
        for (int j = 0; j < ui.nkv; ++j) {
          const uint32_t s = vc % kVS, ph = (vc / kVS) & 1;
          const uint32_t sb = vc % kVBS, phb = (vc / kVBS) & 1;
          if (!mbar_wait_warp(&bars[kBarVFull + s], ph, abort_flag)) { record_failure(abort_flag, kPSiteConvV); ok = false; break; }
          if (!mbar_wait_warp(&bars[kBarVbfEmpty + sb], phb ^ 1, abort_flag)) { record_failure(abort_flag, kPSiteConvE); ok = false; break; }
          const uint8_t* src = smem + L::v + s * kTileBytes + t * 128;
          const uint32_t sfw = reinterpret_cast<const uint32_t*>(smem + L::v_sf + s * kAtomBytes)[(t & 31) * 4 + (t >> 5)];
          uint8_t* dst = smem + L::vbf + sb * kBfTileBytes + t * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c) {  // 16 fp8 values: head_dim [16c, 16c + 16)
            const uint4 raw = *reinterpret_cast<const uint4*>(src + ((static_cast<uint32_t>(c) ^ sw) << 4));
            const int e = static_cast<int>((sfw >> (8 * (c >> 1))) & 0xFFu) - 127;
            const float scale = e >= -126 ? __uint_as_float(static_cast<uint32_t>(e + 127) << 23)
                                          : __uint_as_float(0x00400000u);  // 2^-127
            const uint32_t wv[4] = {raw.x, raw.y, raw.z, raw.w};
            uint32_t outw[8];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const uint32_t h01 = cvt_e4m3x2_to_f16x2(static_cast<uint16_t>(wv[i] & 0xFFFFu));
              const uint32_t h23 = cvt_e4m3x2_to_f16x2(static_cast<uint16_t>(wv[i] >> 16));
              const float2 f01 = __half22float2(*reinterpret_cast<const __half2*>(&h01));
              const float2 f23 = __half22float2(*reinterpret_cast<const __half2*>(&h23));
              outw[2 * i] = cvt_bf16x2(f01.x * scale, f01.y * scale);
              outw[2 * i + 1] = cvt_bf16x2(f23.x * scale, f23.y * scale);
            }
            // bf16 chunks 2c and 2c + 1 (8 elements each): atom a = chunk / 8 holds head_dim
            // [64a, 64a + 64); rows are keys.
#pragma unroll
            for (int hc = 0; hc < 2; ++hc) {
              const uint32_t chunk = 2 * c + hc;
              const uint32_t atom = chunk >> 3, cc = chunk & 7;
              *reinterpret_cast<uint4*>(dst + atom * kBfAtomBytes + ((cc ^ sw) << 4)) =
                  make_uint4(outw[4 * hc], outw[4 * hc + 1], outw[4 * hc + 2], outw[4 * hc + 3]);
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&bars[kBarVbfFull + sb]);
            mbar_arrive(&bars[kBarVEmpty + s]);
          }
          ++vc;
        }
      }
    } else if (kEpi) {
      // ---------------------------------------------------------------- epilogue (warps 12..15)
      // Thread t owns row t of both query tiles (its warp's TMEM lane quarter). Per unit and query
      // tile i: wait until every PV_i is complete and the softmax warpgroup has left its O scale
      // and LSE in shared memory; read O_i from TMEM 32 columns at a time (the last read releases
      // O_i to the next unit's PV), scale, round to BF16 and store the row; store the LSE.
      const int quarter = warp & 3;
      const int row = quarter * 32 + lane;
      const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
      const float2* stats = reinterpret_cast<const float2*>(smem + L::stats);
      uint32_t rc[2] = {0, 0};  // units finished per query tile
      bool ok = true;
      for (int w = blockIdx.x; w < num_units && ok; w += G) {
        const PairUnit ui = pair_unit(p, sched, w);
        if (ui.nkv <= 0) continue;  // the softmax warps wrote the empty-sum rows (or no tile)
        for (int i = 0; i <= ui.has_q1; ++i) {
          // Long waits (a whole unit): sleep between polls, leaving issue slots to the softmax warps.
          if (!wait_role(&bars[kBarOFull + i], rc[i] & 1, abort_flag)) { record_failure(abort_flag, kPSiteEpiO); ok = false; break; }
          if (!wait_role(&bars[kBarStatsFull + i], rc[i] & 1, abort_flag)) { record_failure(abort_flag, kPSiteEpiStats); ok = false; break; }
          ++rc[i];
          tc_fence_after();
          const float2 st = stats[i * kTileM + row];
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars[kBarStatsFree + i]);
          const bool valid = (ui.qtile0 + i) * kTileM + row < ui.q_len;
          const int64_t tok = ui.o_row0 + i * kTileM + row;
          uint4* dst = reinterpret_cast<uint4*>(p.out + (tok * p.heads + ui.h) * 128);
          const uint32_t o_addr = tmem + lane_addr + kColO + i * 128;
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t r[32];
            tmem_ld32_sync(o_addr + c * 32, r);
            if (c == 3) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&bars[kBarOEmpty + i]);
            }
            if (valid) {
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                uint4 v;
                v.x = cvt_bf16x2(__uint_as_float(r[8 * q + 0]) * st.x, __uint_as_float(r[8 * q + 1]) * st.x);
                v.y = cvt_bf16x2(__uint_as_float(r[8 * q + 2]) * st.x, __uint_as_float(r[8 * q + 3]) * st.x);
                v.z = cvt_bf16x2(__uint_as_float(r[8 * q + 4]) * st.x, __uint_as_float(r[8 * q + 5]) * st.x);
                v.w = cvt_bf16x2(__uint_as_float(r[8 * q + 6]) * st.x, __uint_as_float(r[8 * q + 7]) * st.x);
                dst[c * 4 + q] = v;
              }
            }
          }
          if (valid) p.lse[static_cast<int64_t>(ui.h) * p.tq + tok] = st.y;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(*tmem_slot, kTmemCols);
  }
}

}  // namespace pp
}  // namespace lpfa
