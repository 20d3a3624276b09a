// attn_fwd_pp.cuh -- MXFP8 attention forward over pairs of query tiles (8-bit P modes).
//
// Computes what attn_fwd_kernel computes for the two PV modes that keep P in 8 bits: the fp8 PV
// mode (V an unscaled E4M3 cast, implicit dequant scale 1.0; FastVideo #1654 "fp8 PV mode for the
// FA4-FP4 attention path") and the block-scaled MXFP8 PV mode (P and V scaled per 32 keys). Q and
// K are MXFP8 with one E8M0 scale per 32 elements along head_dim (LP-FA4 README, "MXFP8 forward
// and backward"); O is BF16 and the LSE fp32, natural log; absent descales are the literal 1.0f
// on the same code path (vLLM #63232, "Claims").
//
// Work unit: two consecutive 128-row query tiles Q0, Q1 of one (sequence, head) -- the second
// absent when the sequence has an odd number of tiles and this is its last -- against all K/V
// tiles of that sequence. Each softmax warpgroup owns one query tile: its own row reference, its
// own row sums and its own O accumulator, so nothing of the online softmax crosses warpgroups
// (FlashAttention-4's two-tile ping-pong). Every K and V tile loaded serves both query tiles.
//
// Warp roles (512 threads):
//   warp 0        Q/K producer: Q0, Q1 and their scale atoms once per unit, then K tiles + atoms.
//   warp 3        V producer: V tiles (+ token-orientation scale atoms in MXFP8 PV mode).
//   warp 1        TMEM owner and QK issuer: S = Q_i K_j^T (tcgen05.mma kind::mxf8f6f4.block_scale,
//                 M128 N128 K128) into the one S buffer, for i = 0, 1 in turn, each as soon as the
//                 previous S has been read out by its warpgroup.
//   warp 2        PV issuer: O_i += P_i V_j (kind::f8f6f4, or kind::mxf8f6f4.block_scale in MXFP8
//                 PV mode), P_i from TMEM.
//   warps 4..7    softmax of Q0; warps 8..11 softmax of Q1 (one thread per query row).
//   warps 12..15  idle.
//
// TMEM (512 columns): S [0, 128); O_i [128 + 128 i, 256 + 128 i); P_i [384 + 32 i, 416 + 32 i)
// (128 E4M3 keys, 4 per column); Q scale atoms [448 + 8 qstage + 4 i, +4); K scale atoms
// [464 + 4 (kc & 1), +4); MXFP8 PV: P_i's scale atom [472 + 4 i, +4), V's [480 + 4 (vc & 1), +4).
// A single S buffer is what makes room for the block-scaled QK's scale factors next to two O
// accumulators; the warpgroups pass it back and forth, and P has columns of its own, so a
// warpgroup's next S can be computed while its exponentials of the previous tile still run.
#pragma once

#include "attn_fwd.cuh"

namespace lpfa {
namespace pp {

constexpr int kKStages = 5;
constexpr int kVStages = 4;

// P tiles rotate through kPSlots TMEM slots in the order the PV products consume them (tile j of
// a unit: query tile 0, then 1), so a softmax warpgroup storing P waits only for the PV three P
// tiles back, not for its own previous one.
constexpr uint32_t kPSlots = 3;
constexpr uint32_t kColS = 0;
constexpr uint32_t kColO = 128;    // + 128 * i
constexpr uint32_t kColP = 384;    // + 32 * slot
// Scale atoms. fp8 PV: the Q atoms of both tiles per unit stage and the K atoms in two slots, all
// copied into TMEM ahead of the QK that reads them. MXFP8 PV (whose P and V atoms take the rest of
// the columns): one Q and one K slot, copied right before each QK, once the previous QK -- the
// slots' last reader -- is known to have completed.
constexpr uint32_t kColSFA8 = 480;  // + 8 * qstage + 4 * i   (fp8 PV)
constexpr uint32_t kColSFB8 = 496;  // + 4 * (kc & 1)         (fp8 PV)
constexpr uint32_t kColSFA = 480;   // Q scale atom of the QK being issued (MXFP8 PV)
constexpr uint32_t kColSFB = 484;   // K scale atom of the current K tile (MXFP8 PV)
constexpr uint32_t kColSFP = 488;   // + 4 * slot: P scale atom (MXFP8 PV)
constexpr uint32_t kColSFV = 500;   // + 4 * (vc % 3): V scale atom (MXFP8 PV)
static_assert(kColP + 32 * kPSlots <= kColSFA && kColSFB8 + 8 <= kTmemCols && kColSFV + 4 * 3 <= kTmemCols,
              "TMEM columns");

// Shared memory (offsets from a 1024-byte aligned base).
template <bool kMx>
struct Smem {
  static constexpr uint32_t q = 0;                                          // [kQStages][2] tiles
  static constexpr uint32_t k = q + kQStages * 2 * kTileBytes;
  static constexpr uint32_t v = k + kKStages * kTileBytes;
  static constexpr uint32_t q_sf = v + kVStages * kTileBytes;               // [kQStages][2] atoms
  static constexpr uint32_t k_sf = q_sf + kQStages * 2 * kAtomBytes;
  static constexpr uint32_t v_sf = k_sf + kKStages * kAtomBytes;            // MXFP8 PV only
  static constexpr uint32_t p_sf = v_sf + (kMx ? kVStages * kAtomBytes : 0u);  // [kPSlots] P atoms (MXFP8 PV)
  static constexpr uint32_t sched = p_sf + (kMx ? kPSlots * kAtomBytes : 0u);  // n, units, order, prefix
  static constexpr uint32_t bars = sched + ((2 * kMaxSortSeqs + 3) * 4 + 15) / 16 * 16;
  static constexpr uint32_t num_bars = 48;
  static constexpr uint32_t misc = bars + num_bars * 8;                     // tmem base, abort flag
  static constexpr uint32_t total = misc + 64;
};
template <bool kMx> constexpr uint32_t smem_bytes() { return Smem<kMx>::total + 1024; }
static_assert(smem_bytes<true>() <= 227 * 1024 && smem_bytes<false>() <= 227 * 1024, "shared memory");

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
  kBarDrainPV = 42  // PV issuer's own tcgen05 work done
};
static_assert(kKStages <= 6 && kVStages <= 6, "ring barriers");

// Diagnostic sites (g_lpfa_status[1]) of this kernel's waits: 100 + the role's step.
enum PairSite : int {
  kPSiteProducerQ = 101, kPSiteProducerK, kPSiteProducerV, kPSiteMmaQ, kPSiteMmaK, kPSiteMmaS, kPSiteMmaP,
  kPSiteMmaO, kPSiteMmaV, kPSiteSoftS, kPSiteSoftPV, kPSiteSoftO, kPSiteDrain, kPSiteDebugStall, kPSiteTmem
};

// A work unit: query tiles qtile0 and (has_q1) qtile0 + 1 of one (sequence, head).
struct PairUnit {
  int h, seq, qtile0, q_row0, q_len, k_row0, k_len, nkv, sbq, sbk, has_q1;
};

// Unit order in shared memory: sched[0] = n, sched[1] = number of units, then order[kMaxSortSeqs]
// and prefix[kMaxSortSeqs + 1]. For 1 <= n <= kMaxSortSeqs sequences the units are pairs of query
// tiles: sequences by decreasing key-tile count (longest first), each taking heads * ceil(tiles / 2)
// consecutive units, pairs innermost, so that the CTAs running together share one (sequence,
// head)'s K/V through L2 and the static round-robin over the list approximates longest-processing-
// time scheduling. Beyond kMaxSortSeqs sequences (n = 0) every unit is a single tile in the packed
// head-major order (the pairs' prefix would not fit in shared memory).
__device__ __forceinline__ void build_pair_order(const AttnParams& p, int* sched) {
  const int n = p.num_seqs;
  int* s_order = sched + 2;
  int* s_pre = sched + 2 + kMaxSortSeqs;
  if (n > kMaxSortSeqs) {
    if (threadIdx.x == 0) {
      sched[0] = 0;
      sched[1] = p.num_units;  // heads * total query tiles
    }
    __syncthreads();
    return;
  }
  int* s_cost = s_pre;  // key tiles per sequence, before s_pre holds the prefix
  for (int i = threadIdx.x; i < n; i += blockDim.x)
    s_cost[i] = (__ldg(p.cu_k + i + 1) - __ldg(p.cu_k + i) + kTileN - 1) / kTileN;
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
      if (r < n) {
        const int sq = s_order[r];
        const int nt = __ldg(p.so_q + sq + 1) - __ldg(p.so_q + sq);
        v = p.heads * ((nt + 1) >> 1);
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
      sched[1] = carry;
    }
  }
  __syncthreads();
}

__device__ __forceinline__ PairUnit pair_unit(const AttnParams& p, const int* sched, int w) {
  PairUnit u;
  const int n = sched[0];
  if (n > 0) {
    const int* order = sched + 2;
    const int* pre = sched + 2 + kMaxSortSeqs;
    const int r = find_prefix_smem(pre, n, w);
    u.seq = order[r];
    const int sb = __ldg(p.so_q + u.seq);
    const int nt = __ldg(p.so_q + u.seq + 1) - sb;
    const int np = (nt + 1) >> 1;
    const int local = w - pre[r];
    u.h = local / np;
    const int pair = local - u.h * np;
    u.qtile0 = 2 * pair;
    u.sbq = sb + 2 * pair;
    u.has_q1 = (2 * pair + 1 < nt) ? 1 : 0;
  } else {
    u.h = w / p.total_q_tiles;
    const int g = w - u.h * p.total_q_tiles;
    u.seq = find_prefix(p.so_q, p.num_seqs, g);
    u.qtile0 = g - __ldg(p.so_q + u.seq);
    u.sbq = g;
    u.has_q1 = 0;
  }
  const int cq0 = __ldg(p.cu_q + u.seq);
  u.q_row0 = cq0 + u.qtile0 * kTileM;
  u.q_len = __ldg(p.cu_q + u.seq + 1) - cq0;
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
  static_assert(kPv == kPvFp8 || kPv == kPvMx, "8-bit P modes only");
  constexpr bool kMx = kPv == kPvMx;  // block-scaled MXFP8 PV: P and V scaled per 32 keys
  using L = Smem<kMx>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::bars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::misc + 16);
  int* sched_w = reinterpret_cast<int*>(smem + L::sched);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kQStages; ++i) { mbar_init(&bars[kBarQFull + i], 1); mbar_init(&bars[kBarQEmpty + i], 1); }
    for (int i = 0; i < kKStages; ++i) { mbar_init(&bars[kBarKFull + i], 1); mbar_init(&bars[kBarKEmpty + i], 1); }
    for (int i = 0; i < kVStages; ++i) { mbar_init(&bars[kBarVFull + i], 1); mbar_init(&bars[kBarVEmpty + i], 1); }
    mbar_init(&bars[kBarSFree], 4);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars[kBarSFull + i], 1);
      mbar_init(&bars[kBarOFull + i], 1);
      mbar_init(&bars[kBarOEmpty + i], 4);
    }
    for (uint32_t i = 0; i < kPSlots; ++i) {
      // PReady counts the 4 warps of the storing warpgroup; an arrival for the slot's next P
      // needs the PV of this one complete, so the phases of one slot cannot mix.
      mbar_init(&bars[kBarPReady + i], 4);
      mbar_init(&bars[kBarPVDone + i], 1);
    }
    mbar_init(&bars[kBarDrain], 1);
    mbar_init(&bars[kBarDrainPV], 1);
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
        if (ui.nkv == 0) continue;  // no keys: the softmax warps write the empty-sum result
        const uint32_t qs = qc % kQStages, qph = (qc / kQStages) & 1;
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
        for (int j = 0; j < ui.nkv; ++j) {
          const uint32_t s = kc % kKStages, ph = (kc / kKStages) & 1;
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
      for (uint32_t i = (qc > kQStages ? qc - kQStages : 0); i < qc; ++i)
        if (!mbar_wait(&bars[kBarQFull + i % kQStages], (i / kQStages) & 1, nullptr)) record_failure(abort_flag, kPSiteDrain);
      for (uint32_t i = (kc > kKStages ? kc - kKStages : 0); i < kc; ++i)
        if (!mbar_wait(&bars[kBarKFull + i % kKStages], (i / kKStages) & 1, nullptr)) record_failure(abort_flag, kPSiteDrain);
    } else if (warp == 3) {
      // ---------------------------------------------------------------- V producer
      uint32_t vc = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < num_units && ok; w += G) {
        const PairUnit ui = warp_uniform(pair_unit(p, sched, w));
        for (int j = 0; j < ui.nkv; ++j) {
          const uint32_t s = vc % kVStages, ph = (vc / kVStages) & 1;
          if (!wait_role(&bars[kBarVEmpty + s], ph ^ 1, abort_flag)) { record_failure(abort_flag, kPSiteProducerV); ok = false; break; }
          mbar_arrive_expect_tx(&bars[kBarVFull + s], kTileBytes + (kMx ? kAtomBytes : 0u), leader);
          tma_load_3d(smem + L::v + s * kTileBytes, &tmap_v, &bars[kBarVFull + s], 0, ui.h, ui.k_row0 + j * kTileN,
                      leader);
          if (kMx)
            bulk_load(smem + L::v_sf + s * kAtomBytes,
                      p.v_sf + (static_cast<int64_t>(ui.sbk + j) * p.heads + ui.h) * kAtomBytes, kAtomBytes,
                      &bars[kBarVFull + s], leader);
          ++vc;
        }
      }
      for (uint32_t i = (vc > kVStages ? vc - kVStages : 0); i < vc; ++i)
        if (!mbar_wait(&bars[kBarVFull + i % kVStages], (i / kVStages) & 1, nullptr)) record_failure(abort_flag, kPSiteDrain);
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
      for (int w = blockIdx.x; w < num_units && ok; w += G) {
        const PairUnit ui = warp_uniform(pair_unit(p, sched, w));
        if (ui.nkv == 0) continue;
        // The sign of the logit scale goes into the MMA (negated A); the softmax uses |scale|.
        const float qd = descale_value(p.q_descale, ui.seq, ui.h);
        const float kd = descale_value(p.k_descale, ui.seq, ui.h);
        const int negate = (qd * kd) < 0.0f ? 1 : 0;
        uint32_t idq[4];
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) idq[kk] = idesc_qk(kk, negate);
        const uint32_t qs = u % kQStages;
        if (!wait_role(&bars[kBarQFull + qs], (u / kQStages) & 1, abort_flag)) { record_failure(abort_flag, kPSiteMmaQ); ok = false; break; }
        if (!kMx) {
          // fp8 PV: both tiles' Q atoms into this unit stage's slots. Their last reader, the unit
          // two back, completed before the first QK of the previous unit could write S.
          tc_fence_after();
          for (int i = 0; i <= ui.has_q1; ++i)
            tmem_cp_32x128b_x4(tmem + kColSFA8 + qs * 8 + i * 4, dqsf0 + ((qs * 2 + i) * kAtomBytes >> 4), leader);
        }
        // K tile kc is waited for, and (fp8 PV) its atom copied into slot kc & 1, right after the
        // previous tile's last QK has been issued, so that neither sits between the next SFree
        // and the next QK. The slot's last reader, a QK of tile kc - 2, completed before the S
        // that the last SFree released was written.
        auto prepare_k = [&]() -> bool {
          if (!wait_role(&bars[kBarKFull + kc % kKStages], (kc / kKStages) & 1, abort_flag)) return false;
          if (!kMx) {
            tc_fence_after();
            tmem_cp_32x128b_x4(tmem + kColSFB8 + (kc & 1) * 4, dksf0 + ((kc % kKStages) * kAtomBytes >> 4), leader);
          }
          return true;
        };
        if (!prepare_k()) { record_failure(abort_flag, kPSiteMmaK); ok = false; break; }
        for (int j = 0; j < ui.nkv && ok; ++j) {
          const uint32_t s = kc % kKStages;
          const uint64_t bdesc = dk0 + (s * kTileBytes >> 4);
          const uint32_t sfb = tmem + (kMx ? kColSFB : kColSFB8 + (kc & 1) * 4);
          for (int i = 0; i <= ui.has_q1; ++i) {
            if (uses > 0) {
#if LPFA_PP_SFREE_SPIN
              if (!mbar_wait_warp(&bars[kBarSFree], (uses - 1) & 1, abort_flag)) { record_failure(abort_flag, kPSiteMmaS); ok = false; break; }
#else
              if (!wait_role(&bars[kBarSFree], (uses - 1) & 1, abort_flag)) { record_failure(abort_flag, kPSiteMmaS); ok = false; break; }
#endif
            }
            tc_fence_after();
            const uint32_t sfa = tmem + (kMx ? kColSFA : kColSFA8 + qs * 8 + i * 4);
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
      const uint64_t dv0 = umma_desc(sb + L::v, kTileBytes, 1024, kLayoutSw128);
      const uint64_t dpsf0 = umma_desc(sb + L::p_sf, 0, 128, kLayoutNone);
      const uint64_t dvsf0 = umma_desc(sb + L::v_sf, 0, 128, kLayoutNone);
      uint32_t vc = 0;          // V tiles
      uint32_t n = 0;           // P tiles, in the order the PVs consume them
      uint32_t uc[2] = {0, 0};  // units per warpgroup
      bool ok = true;
      for (int w = blockIdx.x; w < num_units && ok; w += G) {
        const PairUnit ui = warp_uniform(pair_unit(p, sched, w));
        if (ui.nkv == 0) continue;
        for (int j = 0; j < ui.nkv && ok; ++j) {
          const uint32_t vs = vc % kVStages;
          // V first: it is loaded well ahead, so this wait is off the path from P to PV.
          if (!wait_role(&bars[kBarVFull + vs], (vc / kVStages) & 1, abort_flag)) { record_failure(abort_flag, kPSiteMmaV); ok = false; break; }
          const uint64_t bdesc = dv0 + (vs * kTileBytes >> 4);
          for (int i = 0; i <= ui.has_q1; ++i) {
            const uint32_t ps = n % kPSlots;
            if (!wait_role(&bars[kBarPReady + ps], (n / kPSlots) & 1, abort_flag)) { record_failure(abort_flag, kPSiteMmaP); ok = false; break; }
            if (j == 0 && !wait_role(&bars[kBarOEmpty + i], (uc[i] & 1) ^ 1, abort_flag)) { record_failure(abort_flag, kPSiteMmaO); ok = false; break; }
            tc_fence_after();
            const uint32_t p_col = tmem + kColP + ps * 32;
            const uint32_t o_col = tmem + kColO + i * 128;
            if (kMx) {
              // Scale atoms into TMEM, in order with the MMAs below: V's once per V tile into slot
              // vc % 3, P's from the softmax's shared-memory atom of this P slot into the matching
              // TMEM slot. Before storing this P the softmax waited for the PV three P tiles
              // back, so every PV that read either slot earlier has completed.
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
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)  // keys [32kk, 32kk + 32): 8 columns of 4 E4M3 each
                mma_f8f6f4_ts(o_col, p_col + kk * 8, bdesc + kk * 256, kIdescPV8, (j > 0 || kk > 0) ? 1u : 0u, leader);
            }
            mma_commit(&bars[kBarPVDone + ps], leader);
            ++n;
          }
          if (!ok) break;
          mma_commit(&bars[kBarVEmpty + vs], leader);
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
    // (Block-scaled P has no E4M3 range limit to respect: it takes the bf16 mode's lag.)
    constexpr float kLag = kMx ? SoftmaxLag<false>::lag : kLagP8;
    constexpr float kBias = kMx ? SoftmaxLag<false>::bias : kBiasP8;
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
    bool ok = true;
    for (int w = blockIdx.x; w < num_units && ok; w += G) {
      const PairUnit ui = pair_unit(p, sched, w);
      const uint32_t np = 1u + static_cast<uint32_t>(ui.has_q1);  // P tiles per key tile
      const uint32_t n0 = nbase;
      nbase += static_cast<uint32_t>(ui.nkv) * np;
      if (grp > ui.has_q1) continue;
      const bool valid = (ui.qtile0 + grp) * kTileM + row < ui.q_len;
      const int64_t tok = ui.q_row0 + grp * kTileM + row;
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
      float m_r = -INFINITY;  // row reference (integer, log2 units)
      float l_r = 0.0f;       // row sum of p (times 2^kBias), relative to m_r
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
        float gmax[4];  // block-scaled MXFP8 P: the 32-key group maxima of S
        float m_new;
        float psum;
        uint32_t mx_sfw = 0;  // block-scaled MXFP8 P: this row's four E8M0 scale bytes
        uint32_t pk[32];      // P as E4M3 codes, four keys per word
        auto no_handoff = [](float) {};
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
          if (tail) exp_row_groups<true>(sv, cscale, nbg, key0, ui.k_len, no_handoff, gsum);
          else exp_row_groups<false>(sv, cscale, nbg, key0, ui.k_len, no_handoff, gsum);
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
          psum = exp_row_e4m3(sv, cscale, kBias - m_new, pk);
        }
        const float m_prev = m_r;
        l_r = l_r * exp2_int(m_prev - m_new) + psum;
        m_r = m_new;
        // This P's slot is free once the PV three P tiles back, its previous reader, has completed.
        const uint32_t n = n0 + static_cast<uint32_t>(j) * np + static_cast<uint32_t>(grp);
        const uint32_t ps = n % kPSlots;
        if (n >= kPSlots) {
          if (!wait_warp(&bars[kBarPVDone + ps], ((n - kPSlots) / kPSlots) & 1, abort_flag, false)) { record_failure(abort_flag, kPSiteSoftPV); ok = false; break; }
          tc_fence_after();
        }
        if (kMx) {
          // The row's four scale bytes go to this warpgroup's shared-memory atom (row r at
          // (r % 32) * 16 + (r / 32) * 4), read by the PV issuer's tcgen05.cp.
          p_sf_words[ps * (kAtomBytes / 4) + (row & 31) * 4 + (row >> 5)] = mx_sfw;
          fence_proxy_async_smem();
        }
        tmem_st32_sync(tmem + lane_addr + kColP + ps * 32, pk);
        // O_i holds tiles up to j - 1 relative to m_prev: rescale it when the reference moved
        // (rare; never on a unit's first tile), once PV_i of tile j - 1 has completed. (That PV's
        // slot cannot have been reused yet: its next use needs this P consumed first.)
        if (j > 0 && __any_sync(0xFFFFFFFFu, m_new != m_prev)) {
          const uint32_t nprev = n - np;
          if (!wait_warp(&bars[kBarPVDone + nprev % kPSlots], (nprev / kPSlots) & 1, abort_flag, false)) { record_failure(abort_flag, kPSiteSoftPV); ok = false; break; }
          tc_fence_after();
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
      // ---------------------------------------------------------------- epilogue
      if (!wait_warp(&bars[kBarOFull + grp], ucnt & 1, abort_flag, false)) { record_failure(abort_flag, kPSiteSoftO); ok = false; break; }
      tc_fence_after();
      const float oscale = descale_value(p.v_descale, ui.seq, ui.h) / l_r;
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
