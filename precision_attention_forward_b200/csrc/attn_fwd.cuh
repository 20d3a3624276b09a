// attn_fwd.cuh -- persistent, warp-specialized MXFP8 attention forward for sm_100a.
//
// Computes, per (sequence, head), O = softmax(Q K^T * qd * kd / sqrt(128)) V * vd and the
// natural-log LSE, for noncausal head_dim 128 over packed variable-length sequences
// (LP-FA4 README, "MXFP8 forward and backward"). Q and K are MXFP8 (E4M3 payload, one E8M0
// scale per 32 elements along head_dim). V is MXFP8 (bf16 PV mode: dequantized to BF16 in
// shared memory, P rounded to BF16), an unscaled E4M3 cast (fp8 PV mode of FastVideo #1654: no
// V scales, implicit dequant scale 1.0, output still BF16), or BF16 that is never quantized
// (bf16 PV with BF16 V, loaded by TMA straight into the BF16 operand layout).
// Absent descales are the literal 1.0f on the same code path (vLLM #63232, "Claims").
//
// Work unit: one 128-row query tile of one (sequence, head). The grid is persistent (one CTA
// per SM); CTA b takes units b, b + G, b + 2G, ... in head-major order so that the CTAs
// running at the same time stream the same K/V through L2.
//
// Warp roles (512 threads, four warpgroups):
//   warp 0        Q/K producer (whole warp, one lane issues TMA): the Q tile + its scale atom
//                 once per unit, then 128-key K tiles + their scale atoms.
//   warp 3        V producer: 128-key V tiles (+ scale atoms in bf16 PV mode).
//   warp 1        TMEM allocator and QK issuer (whole warp, one lane issues):
//                   S[t & 1] = Q K_t^T  tcgen05.mma kind::mxf8f6f4.block_scale, M128 N128 K128
//                 as soon as S buffer t & 1 has been read out by its softmax group.
//   warp 2        PV issuer:  O += P_t V_t  kind::f8f6f4 (fp8 PV) or kind::f16 (bf16 PV), P in
//                 TMEM. Issuing QK and PV from two warps keeps a wait for the softmax from
//                 delaying the next QK, and overlaps one warp's barrier waits with the other's
//                 MMA issue (a tcgen05.mma issue blocks for about as long as the tensor core
//                 needs to execute the previous one).
//   warps 4..7    softmax group 0: KV tiles t with t even (t counts all tiles of the CTA).
//   warps 8..11   softmax group 1: KV tiles t with t odd. In both groups a thread owns one query
//                 row and all 128 keys of the tile (192 registers after setmaxnreg). The groups
//                 run half a tile apart, so one group's exponentials (MUFU) overlap the other's
//                 load, max, packing and stores.
//   warps 12..15  bf16 PV mode with MXFP8 V: convert the V tile to BF16 in shared memory.
//
// Online softmax keeps one reference m per row (an integer, log2 units) shared by the two
// groups: tile t's reference is its own row-maximum ceiling if that exceeds tile t-1's
// reference by more than a lag, else tile t-1's reference, so P <= 2^(lag + bias) and the
// reference (and with it l and O) moves rarely and only by exact powers of two. Tile t-1's
// reference reaches tile t through shared memory after the other group's exponentials. In fp8
// PV mode P is stored as E4M3(2^(bias - m) 2^s) <= 256; the power of two cancels in the final
// division.
//
// TMEM columns (512 allocated): S buffer b at [128b, 128b + 128), O [256, 384), fp8 P slot
// t % 3 at [384 + 32 (t % 3), 416 + 32 (t % 3)) (bf16 P is written over the first 64 columns
// of its S buffer), Q scale atoms (2 stages) [480, 488), K scale atoms (2 slots) [488, 496).
// Three fp8 P slots let a group store P(t) once PV(t - 3) is done; with two, P(t) would wait
// for PV(t - 2), which the tensor pipe is often still executing.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "ptx.cuh"

namespace lpfa {

__device__ int g_lpfa_status[2];  // [0] = lpfa_status code of a failed kernel, [1] = detail

constexpr int kAttnThreads = 512;
constexpr int kLaunchRegs = 128;     // 65536 / 512: registers per thread at launch
constexpr int kSoftmaxRegs = 192;    // softmax warpgroups after setmaxnreg.inc
constexpr int kOtherRegs = 64;       // producer/MMA and converter warpgroups after setmaxnreg.dec
static_assert(2 * kSoftmaxRegs + 2 * kOtherRegs == 4 * kLaunchRegs, "register split must use the launch budget");
constexpr int kTileM = 128;          // query rows per tile
constexpr int kTileN = 128;          // keys per KV tile
constexpr int kQStages = 2;
// K / V / BF16-V ring depths. K tiles are on the QK critical path and their loads see long
// latencies while every SM streams the same head's K/V through L2, so in fp8 PV mode (no
// BF16 V buffers) the shared memory goes to deeper K and V rings.
template <bool kFp8PV> struct Stages;
template <> struct Stages<true> { static constexpr int k = 6, v = 5, vbf = 1; };
template <> struct Stages<false> { static constexpr int k = 3, v = 3, vbf = 2; };
constexpr uint32_t kTileBytes = 128 * 128;     // 128 rows x 128 fp8
constexpr uint32_t kVbfBytes = 128 * 128 * 2;  // 128 keys x 128 bf16
constexpr uint32_t kAtomBytes = 512;

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;        // + 128 * b  S buffer (fp32); bf16 P over its first 64 columns
constexpr uint32_t kColO = 256;      // O accumulator (fp32)
constexpr uint32_t kColP = 384;      // + 32 * (t % kPSlots)  fp8 P slot
constexpr uint32_t kPSlots = 3;
constexpr uint32_t kColSFA = 480;    // + 4 * stage  Q scale atom
constexpr uint32_t kColSFB = 488;    // + 4 * slot   K scale atom
constexpr uint32_t kColSFP = 496;    // + 4 * (t & 1)   P scale atom (block-scaled MXFP8 PV)
constexpr uint32_t kColSFV = 504;    // + 4 * (vc & 1)  V scale atom (block-scaled MXFP8 PV)
static_assert(kColP + 32 * kPSlots <= kColSFA && kColSFV + 8 <= kTmemCols, "TMEM columns");

// log2(e) / sqrt(128) rounded to fp32: logits in log2 units per unit of Q.K.
constexpr float kLog2eRsqrtD = 0.12751743082459868f;
constexpr float kLn2 = 0.69314718055994531f;

// Diagnostic codes stored in g_lpfa_status[1] when a wait gives up.
enum WaitSite : int {
  kSiteProducerQ = 1, kSiteProducerK, kSiteProducerV, kSiteMmaQ, kSiteMmaK, kSiteMmaP,
  kSiteMmaV, kSiteMmaO, kSiteSoftS, kSiteSoftRed, kSiteSoftPV, kSiteSoftL, kSiteConvV,
  kSiteConvE, kSiteDrain, kSiteDebugStall, kSiteMmaS, kSiteSoftO, kSiteTmem
};

// A descale indexed by (sequence, head): ptr[seq * seq_stride + h * head_stride] (vLLM #63232,
// "Claims": per-head scales keep their descale tensors). A missing descale is read as exactly
// 1.0 (same page): the host points it at g_lpfa_one with zero strides, so the kernel always
// loads (no branch on the pointer) and 1.0 takes the same arithmetic path as any other value.
struct Descale {
  const float* ptr;
  int64_t seq_stride, head_stride;
};

__device__ const float g_lpfa_one = 1.0f;

__device__ __forceinline__ float descale_value(const Descale& d, int seq, int h) {
  return __ldg(d.ptr + seq * d.seq_stride + h * d.head_stride);
}

struct AttnParams {
  const uint8_t* q_sf;
  const uint8_t* k_sf;
  const uint8_t* v_sf;      // bf16 PV mode only
  const int32_t* cu_q;      // meta_q.dev
  const int32_t* so_q;      // meta_q.dev + n + 1 (scale / tile prefix)
  const int32_t* cu_k;
  const int32_t* so_k;
  Descale q_descale, k_descale, v_descale;
  __nv_bfloat16* out;       // (Tq, H, 128)
  float* lse;               // (H, Tq)
  int num_seqs;
  int heads;
  int tq;                   // total query tokens
  int total_q_tiles;        // meta_q.total_scale_blocks
  int num_units;            // heads * total_q_tiles
  int debug_stall;          // test hook: >0 makes the MMA warp wait on a phase that never comes
};

// Work order: up to this many sequences are ordered longest first (by key tiles) in shared
// memory at the start of the kernel; beyond it units keep the plain head-major order.
#ifndef LPFA_MAX_SORT_SEQS
#define LPFA_MAX_SORT_SEQS 256
#endif
constexpr int kMaxSortSeqs = LPFA_MAX_SORT_SEQS;

// Shared memory layout (offsets from a 1024-byte aligned base).
template <bool kFp8PV>
struct SmemLayout {
  static constexpr int kK = Stages<kFp8PV>::k, kV = Stages<kFp8PV>::v, kVbf = Stages<kFp8PV>::vbf;
  static constexpr uint32_t q = 0;
  static constexpr uint32_t k = q + kQStages * kTileBytes;
  static constexpr uint32_t v = k + kK * kTileBytes;
  static constexpr uint32_t vbf = v + kV * kTileBytes;                // bf16 PV mode
  static constexpr uint32_t q_sf = vbf + (kFp8PV ? 0 : kVbf * kVbfBytes);
  static constexpr uint32_t k_sf = q_sf + kQStages * kAtomBytes;
  static constexpr uint32_t v_sf = k_sf + kK * kAtomBytes;
  static constexpr uint32_t p_sf = v_sf + kV * kAtomBytes;            // [kPSlots] P scale atoms (MXFP8 PV)
  static constexpr uint32_t mref = p_sf + kPSlots * kAtomBytes;       // float [2 groups][128] tile reference
  static constexpr uint32_t lsum = mref + 2 * 128 * 4;                // float [2 groups][128] partial l
  static constexpr uint32_t mfin = lsum + 2 * 128 * 4;                // float [2 groups][128] reference of l
  static constexpr uint32_t lsumr = mfin + 2 * 128 * 4;               // float [2 groups][128] partial sum of rounded P
  static constexpr uint32_t sched = lsumr + 2 * 128 * 4;              // int: n, order[kMaxSortSeqs], prefix[kMaxSortSeqs + 1]
  static constexpr uint32_t bars = sched + ((2 * kMaxSortSeqs + 2) * 4 + 15) / 16 * 16;  // uint64 barriers
  static constexpr uint32_t num_bars = 64;
  static constexpr uint32_t misc = bars + num_bars * 8;               // tmem base, abort flag
  static constexpr uint32_t total = misc + 64;
};
template <bool kFp8PV> constexpr uint32_t attn_smem_bytes() { return SmemLayout<kFp8PV>::total + 1024; }  // + alignment slack
static_assert(attn_smem_bytes<true>() <= 227 * 1024 && attn_smem_bytes<false>() <= 227 * 1024, "shared memory");

// Barrier indices. [2]-sized entries are indexed by softmax group / S buffer b.
enum Bar : int {
  kBarQFull = 0, kBarQEmpty = 2,         // [kQStages]
  kBarKFull = 4, kBarKEmpty = 10,        // [up to 6]
  kBarVFull = 16, kBarVEmpty = 22,       // [up to 6]
  kBarVbfFull = 28, kBarVbfEmpty = 30,   // [2]
  kBarSFull = 32,    // S(t) computed                       (MMA commit)
  kBarSFree = 34,    // S(t) read out by its group            (4 warps)
  kBarPReady = 36,   // [t % kPSlots] P(t) stored, O rescaled if needed (4 warps)
  kBarPVDone = 39,   // [t % kPSlots] PV(t) complete           (MMA commit)
  kBarOFull = 42,    // every PV of the unit complete         (MMA commit)
  kBarOEmpty = 43,   // O read out by both groups             (8 warps)
  kBarLReady = 44,   // partial l / reference exchanged       (8 warps)
  kBarDrain = 45,    // QK issuer's own tcgen05 work done
  kBarDrainPV = 46,  // PV issuer's own tcgen05 work done
  kBarMRef = 48      // [group][lane quarter]: tile reference of t published and the MUFU
                     // handed over to the other group (1 warp; 8 entries)
};
static_assert(Stages<true>::k <= 6 && Stages<true>::v <= 6 && Stages<false>::k <= 6 && Stages<false>::v <= 6, "ring barriers");

// UMMA shared-memory matrix descriptor (sm_100 format, version 1).
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
  return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4) |
         (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) |
         (1ull << 46) | (static_cast<uint64_t>(layout) << 61);
}
constexpr uint32_t kLayoutSw128 = 2;
constexpr uint32_t kLayoutNone = 0;

// Instruction descriptors.
// Block-scaled E4M3 x E4M3 -> F32, M=128, N=128, both operands K-major, E8M0 scales.
__device__ __forceinline__ uint32_t idesc_qk(int kb, int negate_a) {
  return (static_cast<uint32_t>(kb) << 4) | (static_cast<uint32_t>(negate_a) << 13) |
         ((kTileN >> 3) << 17) | (1u << 23) | (8u << 24) | (static_cast<uint32_t>(kb) << 29);
}
// E4M3 x E4M3 -> F32, M=128, N=128, A (P) K-major in TMEM, B (V) MN-major.
constexpr uint32_t kIdescPV8 = (1u << 4) | (1u << 16) | (16u << 17) | (8u << 24);
// Block-scaled E4M3 x E4M3 -> F32, M=128, N=128, A (P) K-major in TMEM, B (V) MN-major, E8M0
// scales; kb selects the scale byte of the K step (keys [32kb, 32kb + 32)).
__device__ __forceinline__ uint32_t idesc_pv_mx(int kb) {
  return (static_cast<uint32_t>(kb) << 4) | (1u << 16) | ((128u >> 3) << 17) | (1u << 23) | (8u << 24) |
         (static_cast<uint32_t>(kb) << 29);
}
// BF16 x BF16 -> F32, M=128, N=128, A (P) K-major in TMEM, B (V) MN-major.
constexpr uint32_t kIdescPV16 = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | (16u << 17) | (8u << 24);

// ---------------------------------------------------------------------------------------
// Softmax helpers (one thread = one query row, the 128 keys of an S tile held as 64 float2)
// ---------------------------------------------------------------------------------------
// Pairs of S elements, out of every 8, whose exp2 runs on the FMA pipe (polynomial) instead
// of the MUFU unit. MUFU alone delivers 16 exp2 per clock per SM, half of what the FP8 tensor
// core would need; moving part of the work to the FMA pipe balances the two.
#ifndef LPFA_POLY_PAIRS
#define LPFA_POLY_PAIRS 0
#endif
constexpr int kPolyPairs = LPFA_POLY_PAIRS;

// 2^f on [-0.5, 0.5]: minimax-in-relative-error cubic, float32 coefficients produced by
// csrc/exp2_poly_fit.py (max relative error 7.5e-5 in float32 Horner form).
constexpr float kExp2P0 = 0.9999280571937561f;
constexpr float kExp2P1 = 0.6932609677314758f;
constexpr float kExp2P2 = 0.2426111251115799f;
constexpr float kExp2P3 = 0.0551716685295105f;

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// 2^k for an integer-valued k <= 0 (or -inf), exactly; 0 below the normal range.
__device__ __forceinline__ float exp2_int(float k) {
  return k < -126.0f ? 0.0f : __uint_as_float(static_cast<uint32_t>(static_cast<int>(k) + 127) << 23);
}

__device__ __forceinline__ float2 exp2_mufu2(float2 x) {
  return make_float2(ex2_approx(x.x), ex2_approx(x.y));
}

// 2^x = 2^j * q(x - j), j = round(x) by the 1.5 * 2^23 magic add; the exponent of q is
// raised by j with one integer add on the bit pattern. Inputs below -126 (a masked key's -inf
// included) give exactly 0, as the MUFU exponential does.
__device__ __forceinline__ float2 exp2_poly2(float2 xin) {
  float2 x;
  x.x = fmaxf(xin.x, -126.0f);
  x.y = fmaxf(xin.y, -126.0f);
  const float2 t = __fadd2_rn(x, make_float2(12582912.0f, 12582912.0f));
  const float2 jf = __fadd2_rn(t, make_float2(-12582912.0f, -12582912.0f));
  const float2 f = __ffma2_rn(jf, make_float2(-1.0f, -1.0f), x);
  float2 q = __ffma2_rn(make_float2(kExp2P3, kExp2P3), f, make_float2(kExp2P2, kExp2P2));
  q = __ffma2_rn(q, f, make_float2(kExp2P1, kExp2P1));
  q = __ffma2_rn(q, f, make_float2(kExp2P0, kExp2P0));
  const float2 r = make_float2(__uint_as_float(__float_as_uint(q.x) + (__float_as_uint(t.x) << 23)),
                               __uint_as_float(__float_as_uint(q.y) + (__float_as_uint(t.y) << 23)));
  return make_float2(xin.x < -126.0f ? 0.0f : r.x, xin.y < -126.0f ? 0.0f : r.y);
}

// The 128 S columns of this thread's row.
__device__ __forceinline__ void load_row(uint32_t taddr, float2 (&s)[64]) {
  uint32_t r[128];
  tmem_ld128_sync(taddr, r);
#pragma unroll
  for (int i = 0; i < 64; ++i) s[i] = make_float2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
}

__device__ __forceinline__ void mask_keys(float2 (&s)[64], int key0, int klen) {
#pragma unroll
  for (int i = 0; i < 64; ++i) {
    if (key0 + 2 * i >= klen) s[i].x = -INFINITY;
    if (key0 + 2 * i + 1 >= klen) s[i].y = -INFINITY;
  }
}

__device__ __forceinline__ float rowmax128(const float2 (&s)[64]) {
  float a[16];
#pragma unroll
  for (int k = 0; k < 16; ++k)
    a[k] = max3f(max3f(s[4 * k].x, s[4 * k].y, s[4 * k + 1].x), max3f(s[4 * k + 1].y, s[4 * k + 2].x, s[4 * k + 2].y),
                 fmaxf(s[4 * k + 3].x, s[4 * k + 3].y));
  const float b0 = max3f(a[0], a[1], a[2]), b1 = max3f(a[3], a[4], a[5]), b2 = max3f(a[6], a[7], a[8]);
  const float b3 = max3f(a[9], a[10], a[11]), b4 = max3f(a[12], a[13], a[14]);
  return fmaxf(max3f(b0, b1, b2), max3f(b3, b4, a[15]));
}

// rowmax128 that also returns the maxima of the four 32-key groups (16 pairs each).
__device__ __forceinline__ float rowmax128_groups(const float2 (&s)[64], float (&gmax)[4]) {
  float a[16];
#pragma unroll
  for (int k = 0; k < 16; ++k)
    a[k] = max3f(max3f(s[4 * k].x, s[4 * k].y, s[4 * k + 1].x), max3f(s[4 * k + 1].y, s[4 * k + 2].x, s[4 * k + 2].y),
                 fmaxf(s[4 * k + 3].x, s[4 * k + 3].y));
#pragma unroll
  for (int g = 0; g < 4; ++g) gmax[g] = fmaxf(max3f(a[4 * g], a[4 * g + 1], a[4 * g + 2]), a[4 * g + 3]);
  return max3f(max3f(gmax[0], gmax[1], gmax[2]), gmax[3], gmax[3]);
}

// How many of a row's 64 exponential pairs are issued before a softmax group hands the MUFU
// over to the other group (see the softmax loop). Handing over a little before the end
// hides the hand-over latency behind the last exponentials.
#ifndef LPFA_HANDOFF_PAIRS
#define LPFA_HANDOFF_PAIRS 40
#endif
constexpr int kHandoffPairs = LPFA_HANDOFF_PAIRS;
static_assert(kHandoffPairs >= 1 && kHandoffPairs <= 64, "hand-over point out of range");

// p = 2^(s * c + nb) in place; masked keys (tail tiles) become exactly 0. Returns sum of p.
// Written in passes (exponents, exponentials, sum) so that the MUFU operations issue back to
// back at the MUFU rate. handoff(x) runs after the first kHandoffPairs pairs, with x one of
// their results (a data dependency that keeps it from being scheduled earlier).
template <bool kTail, int kPoly, typename F>
__device__ __forceinline__ float exp_row(float2 (&s)[64], float c, float nb, int key0, int klen, F&& handoff) {
  const float2 c2 = make_float2(c, c), nb2 = make_float2(nb, nb);
#pragma unroll
  for (int i = 0; i < 64; ++i) s[i] = __ffma2_rn(s[i], c2, nb2);
#pragma unroll
  for (int i = 0; i < kHandoffPairs; ++i) s[i] = ((i & 7) < kPoly) ? exp2_poly2(s[i]) : exp2_mufu2(s[i]);
  handoff(s[kHandoffPairs - 1].y);
#pragma unroll
  for (int i = kHandoffPairs; i < 64; ++i) s[i] = ((i & 7) < kPoly) ? exp2_poly2(s[i]) : exp2_mufu2(s[i]);
  if (kTail) {
#pragma unroll
    for (int i = 0; i < 64; ++i) {
      if (key0 + 2 * i >= klen) s[i].x = 0.0f;
      if (key0 + 2 * i + 1 >= klen) s[i].y = 0.0f;
    }
  }
  float2 acc[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) acc[k] = s[k];
#pragma unroll
  for (int i = 8; i < 64; ++i) acc[i & 7] = __fadd2_rn(acc[i & 7], s[i]);
  const float2 t0 = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
  const float2 t1 = __fadd2_rn(__fadd2_rn(acc[4], acc[5]), __fadd2_rn(acc[6], acc[7]));
  const float2 t = __fadd2_rn(t0, t1);
  return t.x + t.y;
}

// exp_row for block-scaled MXFP8 P: group g (pairs [16g, 16g + 16)) uses its own bias nbg[g]
// = nb - e_g, so the exponentials come out already scaled by the group's 2^-e_g (an integer
// shift of the exponent). gsum[g] receives the sum of the group's scaled p.
template <bool kTail, typename F>
__device__ __forceinline__ void exp_row_groups(float2 (&s)[64], float c, const float (&nbg)[4], int key0, int klen,
                                               F&& handoff, float (&gsum)[4]) {
  const float2 c2 = make_float2(c, c);
#pragma unroll
  for (int i = 0; i < 64; ++i) s[i] = __ffma2_rn(s[i], c2, make_float2(nbg[i >> 4], nbg[i >> 4]));
#pragma unroll
  for (int i = 0; i < kHandoffPairs; ++i) s[i] = exp2_mufu2(s[i]);
  handoff(s[kHandoffPairs - 1].y);
#pragma unroll
  for (int i = kHandoffPairs; i < 64; ++i) s[i] = exp2_mufu2(s[i]);
  if (kTail) {
#pragma unroll
    for (int i = 0; i < 64; ++i) {
      if (key0 + 2 * i >= klen) s[i].x = 0.0f;
      if (key0 + 2 * i + 1 >= klen) s[i].y = 0.0f;
    }
  }
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    float2 acc[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) acc[k] = s[16 * g + k];
#pragma unroll
    for (int i = 16 * g + 4; i < 16 * g + 16; ++i) acc[i & 3] = __fadd2_rn(acc[i & 3], s[i]);
    const float2 t = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
    gsum[g] = t.x + t.y;
  }
}

struct UnitInfo {
  int h, seq, qtile, q_row0, q_len, k_row0, k_len, nkv, sbq, sbk;
};

__device__ __forceinline__ int find_prefix(const int32_t* prefix, int n, int g) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(prefix + mid) <= g) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Unit order, kept in shared memory (sched[0] = n, sched[1 ..] = order, then the prefix) so that
// nothing of it stays live in registers across the hot loops. Sorted (n > 0): sequences by
// decreasing key-tile count, each taking heads * its query tiles consecutive units, query tiles
// innermost so that the CTAs running together share one (sequence, head)'s K/V through L2; a
// static round-robin over this longest-first list approximates longest-processing-time
// scheduling. Unsorted (n = 0): unit w is head w / total_q_tiles, query tile w % total_q_tiles
// of the packed order.
__device__ __forceinline__ int find_prefix_smem(const int* prefix, int n, int g) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= g) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ UnitInfo unit_info(const AttnParams& p, const int* sched, int w) {
  UnitInfo u;
  const int n = sched[0];
  if (n > 0) {
    const int* order = sched + 1;
    const int* pre = sched + 1 + kMaxSortSeqs;
    const int r = find_prefix_smem(pre, n, w);
    u.seq = order[r];
    u.sbq = __ldg(p.so_q + u.seq);
    const int nq = __ldg(p.so_q + u.seq + 1) - u.sbq;
    const int local = w - pre[r];
    u.h = local / nq;
    u.qtile = local - u.h * nq;
  } else {
    u.h = w / p.total_q_tiles;
    const int g = w - u.h * p.total_q_tiles;
    u.seq = find_prefix(p.so_q, p.num_seqs, g);
    u.sbq = __ldg(p.so_q + u.seq);
    u.qtile = g - u.sbq;
  }
  const int cq0 = __ldg(p.cu_q + u.seq);
  u.q_row0 = cq0 + u.qtile * kTileM;
  u.q_len = __ldg(p.cu_q + u.seq + 1) - cq0;
  u.k_row0 = __ldg(p.cu_k + u.seq);
  u.k_len = __ldg(p.cu_k + u.seq + 1) - u.k_row0;
  u.nkv = (u.k_len + kTileN - 1) / kTileN;
  u.sbk = __ldg(p.so_k + u.seq);
  return u;
}

// Builds the longest-first order in shared memory (all threads of the CTA; ends synchronized).
// More than kMaxSortSeqs sequences, or a single one, keep the plain order (n = 0).
__device__ __forceinline__ void build_unit_order(const AttnParams& p, int* sched) {
  const int n = p.num_seqs;
  int* s_order = sched + 1;
  int* s_pre = sched + 1 + kMaxSortSeqs;
  if (n > kMaxSortSeqs || n < 2) {
    if (threadIdx.x == 0) sched[0] = 0;
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
  // Prefix of heads * query tiles over the sorted sequences (warp 0, 32 at a time).
  if (threadIdx.x < 32) {
    int carry = 0;
    for (int base = 0; base < n; base += 32) {
      const int r = base + static_cast<int>(threadIdx.x);
      int v = 0;
      if (r < n) {
        const int sq = s_order[r];
        v = p.heads * (__ldg(p.so_q + sq + 1) - __ldg(p.so_q + sq));
      }
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int o = __shfl_up_sync(0xFFFFFFFFu, v, d);
        if (threadIdx.x >= static_cast<unsigned>(d)) v += o;
      }
      if (r < n) s_pre[r + 1] = carry + v;     // inclusive prefix -> entry r + 1
      carry += __shfl_sync(0xFFFFFFFFu, v, 31);
    }
    if (threadIdx.x == 0) {
      s_pre[0] = 0;
      sched[0] = n;
    }
  }
  __syncthreads();
}

// Warp-uniform copies of values that every lane of a warp computes identically. Results of
// warp votes and reductions live in uniform registers, which lets the compiler keep the
// producer and MMA loops (trip counts, stage indices, descriptors) on the uniform datapath;
// otherwise every tcgen05.mma operand would need a per-instruction register conversion.
__device__ __forceinline__ int warp_uniform(int x) {
  return static_cast<int>(__reduce_max_sync(0xFFFFFFFFu, static_cast<unsigned>(x)));
}

__device__ __forceinline__ UnitInfo warp_uniform(const UnitInfo& u) {
  UnitInfo r;
  r.h = warp_uniform(u.h);
  r.seq = warp_uniform(u.seq);
  r.qtile = warp_uniform(u.qtile);
  r.q_row0 = warp_uniform(u.q_row0);
  r.q_len = warp_uniform(u.q_len);
  r.k_row0 = warp_uniform(u.k_row0);
  r.k_len = warp_uniform(u.k_len);
  r.nkv = warp_uniform(u.nkv);
  r.sbq = warp_uniform(u.sbq);
  r.sbk = warp_uniform(u.sbk);
  return r;
}

// mbar_wait by a whole warp, with a warp-uniform result.
__device__ __forceinline__ bool mbar_wait_warp(uint64_t* bar, uint32_t parity, const volatile int* abort) {
  return __all_sync(0xFFFFFFFFu, mbar_wait(bar, parity, abort));
}

__device__ __forceinline__ void record_failure(volatile int* abort_flag, int site) {
  *abort_flag = 1;
  if (atomicCAS(&g_lpfa_status[0], 0, 4 /* LPFA_ERR_TIMEOUT */) == 0) atomicExch(&g_lpfa_status[1], site);
}

// PV variants of the kernel: V as MXFP8 dequantized to BF16 in shared memory (bf16 PV), V as
// unscaled E4M3 (fp8 PV), or V given as BF16 and loaded by TMA straight into the layout the
// BF16 PV MMA reads (bf16 PV with BF16 V; LP-FA4 README: the BF16 V path).
enum PvKind : int { kPvBf16Mx = 0, kPvFp8 = 1, kPvBf16In = 2, kPvMx = 3 };
// P as 8-bit codes in the TMEM P slots and V used straight from its 8-bit tile: the fp8 PV mode
// and the block-scaled MXFP8 PV mode share the shared-memory layout and stage counts.
template <int kPv> constexpr bool pv_p8() { return kPv == kPvFp8 || kPv == kPvMx; }

// How far (log2 units) a row's logits may exceed its reference before the reference, l and
// O move, and the power of two P is stored with. bf16 P keeps its 8-bit mantissa at any
// scale, so it may lag 8 binades; fp8 P stores 2^(bias - m) 2^s <= 2^(lag + bias) = 256 < 448.
template <bool kFp8PV> struct SoftmaxLag;
template <> struct SoftmaxLag<true> { static constexpr float lag = 2.0f; static constexpr float bias = 6.0f; };
template <> struct SoftmaxLag<false> { static constexpr float lag = 8.0f; static constexpr float bias = 0.0f; };


// kPerUnitDescale: q/k descales that vary with (sequence, head) are read per unit by the softmax
// (the QK issuer always reads them per unit). The host takes it only when a q or k descale has a
// nonzero stride: reading the scale per unit costs the softmax loop several percent.
template <int kPv, bool kPerUnitDescale>
__global__ void __launch_bounds__(kAttnThreads, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                const __grid_constant__ CUtensorMap tmap_v, const AttnParams p) {
  constexpr bool kFp8PV = kPv == kPvFp8;
  constexpr bool kMx = kPv == kPvMx;        // block-scaled MXFP8 PV: P and V scaled per 32 keys
  constexpr bool kP8 = pv_p8<kPv>();        // P in the TMEM P slots, V from its 8-bit tile
  constexpr bool kVIn = kPv == kPvBf16In;  // BF16 V straight into the BF16 operand buffers
  constexpr bool kVsf = kPv == kPvBf16Mx || kMx;  // V tiles come with a scale atom
  using L = SmemLayout<kP8>;
  constexpr int kKStages = Stages<kP8>::k, kVStages = Stages<kP8>::v, kVbfStages = Stages<kP8>::vbf;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::bars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::misc + 16);
  float* mref = reinterpret_cast<float*>(smem + L::mref);
  float* lsum = reinterpret_cast<float*>(smem + L::lsum);
  float* mfin = reinterpret_cast<float*>(smem + L::mfin);
  float* lsumr = reinterpret_cast<float*>(smem + L::lsumr);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kQStages; ++i) { mbar_init(&bars[kBarQFull + i], 1); mbar_init(&bars[kBarQEmpty + i], 1); }
    for (int i = 0; i < kKStages; ++i) { mbar_init(&bars[kBarKFull + i], 1); mbar_init(&bars[kBarKEmpty + i], 1); }
    for (int i = 0; i < kVStages; ++i) {
      mbar_init(&bars[kBarVFull + i], 1);
      mbar_init(&bars[kBarVEmpty + i], kP8 ? 1 : 4);   // MMA commit, or the 4 converter warps
    }
    for (int i = 0; i < kVbfStages; ++i) {
      mbar_init(&bars[kBarVbfFull + i], kVIn ? 1 : 4);  // the V producer's TMA, or the 4 converter warps
      mbar_init(&bars[kBarVbfEmpty + i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars[kBarSFull + i], 1);
      mbar_init(&bars[kBarSFree + i], 4);
    }
    // PReady and PVDone are indexed by t % kPSlots. PReady counts the 4 warps of a group, which
    // run independently of each other: a warp's arrival for tile t + 3 on the same barrier
    // needs PV(t) complete (the P-slot wait), and so every arrival for tile t, which keeps the
    // phases apart. (One barrier per group would let a fast warp's arrival for t + 2 complete
    // the phase of t before a slow warp had stored its rows of P(t).)
    for (uint32_t i = 0; i < kPSlots; ++i) {
      mbar_init(&bars[kBarPReady + i], 4);
      mbar_init(&bars[kBarPVDone + i], 1);
    }
    mbar_init(&bars[kBarOFull], 1);
    mbar_init(&bars[kBarOEmpty], 8);
    mbar_init(&bars[kBarLReady], 8);
    mbar_init(&bars[kBarDrain], 1);
    mbar_init(&bars[kBarDrainPV], 1);
    for (int i = 0; i < 8; ++i) mbar_init(&bars[kBarMRef + i], 1);
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
  build_unit_order(p, reinterpret_cast<int*>(smem + L::sched));
  const int* sched = reinterpret_cast<const int*>(smem + L::sched);
  // All 512 columns of the SM's tensor memory belong to this CTA (one CTA per SM), so the
  // allocation starts at lane 0, column 0. Using the constant keeps every TMEM operand of
  // the tcgen05 instructions a compile-time or warp-uniform value.
  constexpr uint32_t tmem = 0;
  const bool tmem_ok = *tmem_slot == tmem;
  if (!tmem_ok && threadIdx.x == 0) record_failure(abort_flag, kSiteTmem);

  const int G = gridDim.x;

  if (!tmem_ok) {
    // nothing issued; fall through to the teardown
  } else if (warp < 4) {
    setmaxnreg_dec<kOtherRegs>();
    if (warp == 0) {
      // ---------------------------------------------------------------- Q/K producer
      // The whole warp runs the loop (warp-uniform state); lane 0 issues the copies.
      const uint32_t leader = lane == 0 ? 1u : 0u;
      uint32_t qc = 0, kc = 0;  // fills issued per ring
      bool ok = true;
      for (int w = blockIdx.x; w < p.num_units && ok; w += G) {
        const UnitInfo ui = warp_uniform(unit_info(p, sched, w));
        if (ui.nkv == 0) continue;  // no keys: the softmax warps write the empty-sum result
        const uint32_t qs = qc % kQStages, qph = (qc / kQStages) & 1;
        if (!mbar_wait_warp(&bars[kBarQEmpty + qs], qph ^ 1, abort_flag)) { record_failure(abort_flag, kSiteProducerQ); ok = false; break; }
        mbar_arrive_expect_tx(&bars[kBarQFull + qs], kTileBytes + kAtomBytes, leader);
        tma_load_3d(smem + L::q + qs * kTileBytes, &tmap_q, &bars[kBarQFull + qs], 0, ui.h, ui.q_row0, leader);
        bulk_load(smem + L::q_sf + qs * kAtomBytes,
                  p.q_sf + (static_cast<int64_t>(ui.sbq + ui.qtile) * p.heads + ui.h) * kAtomBytes, kAtomBytes,
                  &bars[kBarQFull + qs], leader);
        ++qc;
        for (int j = 0; j < ui.nkv; ++j) {
          const uint32_t s = kc % kKStages, ph = (kc / kKStages) & 1;
          if (!mbar_wait_warp(&bars[kBarKEmpty + s], ph ^ 1, abort_flag)) { record_failure(abort_flag, kSiteProducerK); ok = false; break; }
          mbar_arrive_expect_tx(&bars[kBarKFull + s], kTileBytes + kAtomBytes, leader);
          tma_load_3d(smem + L::k + s * kTileBytes, &tmap_k, &bars[kBarKFull + s], 0, ui.h,
                      ui.k_row0 + j * kTileN, leader);
          bulk_load(smem + L::k_sf + s * kAtomBytes,
                    p.k_sf + (static_cast<int64_t>(ui.sbk + j) * p.heads + ui.h) * kAtomBytes, kAtomBytes,
                    &bars[kBarKFull + s], leader);
          ++kc;
        }
      }
      // Drain: every copy issued here must land before the CTA exits. The newest fill of each
      // stage is the last one issued into it; older fills of that stage were consumed already.
      for (uint32_t i = (qc > kQStages ? qc - kQStages : 0); i < qc; ++i)
        if (!mbar_wait(&bars[kBarQFull + i % kQStages], (i / kQStages) & 1, nullptr)) record_failure(abort_flag, kSiteDrain);
      for (uint32_t i = (kc > kKStages ? kc - kKStages : 0); i < kc; ++i)
        if (!mbar_wait(&bars[kBarKFull + i % kKStages], (i / kKStages) & 1, nullptr)) record_failure(abort_flag, kSiteDrain);
    } else if (warp == 3 && kVIn) {
      // ---------------------------------------------------------------- V producer (BF16 V)
      // Two TMA box loads per tile (head_dim [0, 64) and [64, 128), 128 keys each, 128-byte
      // swizzle) produce exactly the MN-major BF16 operand layout the PV MMA reads.
      const uint32_t leader = lane == 0 ? 1u : 0u;
      uint32_t vc = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < p.num_units && ok; w += G) {
        const UnitInfo ui = warp_uniform(unit_info(p, sched, w));
        for (int j = 0; j < ui.nkv; ++j) {
          const uint32_t sb = vc % kVbfStages, phb = (vc / kVbfStages) & 1;
          if (!mbar_wait_warp(&bars[kBarVbfEmpty + sb], phb ^ 1, abort_flag)) { record_failure(abort_flag, kSiteProducerV); ok = false; break; }
          mbar_arrive_expect_tx(&bars[kBarVbfFull + sb], kVbfBytes, leader);
#pragma unroll
          for (int a = 0; a < 2; ++a)
            tma_load_3d(smem + L::vbf + sb * kVbfBytes + a * kTileBytes, &tmap_v, &bars[kBarVbfFull + sb], a * 64,
                        ui.h, ui.k_row0 + j * kTileN, leader);
          ++vc;
        }
      }
      for (uint32_t i = (vc > kVbfStages ? vc - kVbfStages : 0); i < vc; ++i)
        if (!mbar_wait(&bars[kBarVbfFull + i % kVbfStages], (i / kVbfStages) & 1, nullptr)) record_failure(abort_flag, kSiteDrain);
    } else if (warp == 3) {
      // ---------------------------------------------------------------- V producer
      // A warp of its own, so that K loads (and with them QK) never wait behind a V stage
      // that the PV of a slower softmax tile still holds.
      const uint32_t leader = lane == 0 ? 1u : 0u;
      uint32_t vc = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < p.num_units && ok; w += G) {
        const UnitInfo ui = warp_uniform(unit_info(p, sched, w));
        for (int j = 0; j < ui.nkv; ++j) {
          const uint32_t s = vc % kVStages, ph = (vc / kVStages) & 1;
          if (!mbar_wait_warp(&bars[kBarVEmpty + s], ph ^ 1, abort_flag)) { record_failure(abort_flag, kSiteProducerV); ok = false; break; }
          mbar_arrive_expect_tx(&bars[kBarVFull + s], kTileBytes + (kVsf ? kAtomBytes : 0), leader);
          tma_load_3d(smem + L::v + s * kTileBytes, &tmap_v, &bars[kBarVFull + s], 0, ui.h,
                      ui.k_row0 + j * kTileN, leader);
          if (kVsf)
            bulk_load(smem + L::v_sf + s * kAtomBytes,
                      p.v_sf + (static_cast<int64_t>(ui.sbk + j) * p.heads + ui.h) * kAtomBytes, kAtomBytes,
                      &bars[kBarVFull + s], leader);
          ++vc;
        }
      }
      for (uint32_t i = (vc > kVStages ? vc - kVStages : 0); i < vc; ++i)
        if (!mbar_wait(&bars[kBarVFull + i % kVStages], (i / kVStages) & 1, nullptr)) record_failure(abort_flag, kSiteDrain);
    } else if (warp == 1) {
      // ---------------------------------------------------------------- QK issuer
      // S(t) = Q K_t^T into S buffer t & 1. The whole warp runs the loop (warp-uniform state);
      // lane 0 issues the tcgen05 instructions.
      const uint32_t leader = lane == 0 ? 1u : 0u;
      // Descriptor bases; the start-address field is the low 14 bits (address >> 4), so a byte
      // offset b inside shared memory advances a descriptor by b >> 4.
      const uint32_t sb = static_cast<uint32_t>(warp_uniform(static_cast<int>(smem_u32(smem))));
      const uint64_t dq0 = umma_desc(sb + L::q, 16, 1024, kLayoutSw128);
      const uint64_t dk0 = umma_desc(sb + L::k, 16, 1024, kLayoutSw128);
      const uint64_t dqsf0 = umma_desc(sb + L::q_sf, 0, 128, kLayoutNone);
      const uint64_t dksf0 = umma_desc(sb + L::k_sf, 0, 128, kLayoutNone);
      uint32_t u = 0, kc = 0, t = 0;  // units, K fills, tiles
      bool ok = true;
      if (p.debug_stall > 0) {
        // Test hook: wait for a phase of the drain barrier that nothing completes before the
        // drains below, so the wait runs out and the failure path is exercised.
        if (!mbar_wait_warp(&bars[kBarDrain], 0, abort_flag)) { record_failure(abort_flag, kSiteDebugStall); ok = false; }
      }
      for (int w = blockIdx.x; w < p.num_units && ok; w += G) {
        const UnitInfo ui = warp_uniform(unit_info(p, sched, w));
        if (ui.nkv == 0) continue;
        // The sign of the logit scale goes into the MMA (negated A); the softmax uses |scale|.
        const float qd = descale_value(p.q_descale, ui.seq, ui.h);
        const float kd = descale_value(p.k_descale, ui.seq, ui.h);
        const int negate = (qd * kd) < 0.0f ? 1 : 0;
        uint32_t idq[4];
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) idq[kk] = idesc_qk(kk, negate);
        const uint32_t qs = u % kQStages;
        if (!mbar_wait_warp(&bars[kBarQFull + qs], (u / kQStages) & 1, abort_flag)) { record_failure(abort_flag, kSiteMmaQ); ok = false; break; }
        tc_fence_after();
        const uint32_t sfa = tmem + kColSFA + qs * 4;
        tmem_cp_32x128b_x4(sfa, dqsf0 + (qs * kAtomBytes >> 4), leader);
        const uint64_t adesc = dq0 + (qs * kTileBytes >> 4);
        for (int j = 0; j < ui.nkv; ++j, ++t) {
          const uint32_t b = t & 1;
          if (t >= 2) {
            // S buffer b has been read out by its group (tile t - 2); in bf16 PV mode it also
            // holds P(t - 2), so PV(t - 2) must have completed.
            if (!mbar_wait_warp(&bars[kBarSFree + b], ((t - 2) >> 1) & 1, abort_flag)) { record_failure(abort_flag, kSiteMmaS); ok = false; break; }
            if (!kP8 && !mbar_wait_warp(&bars[kBarPVDone + (t - 2) % kPSlots], ((t - 2) / kPSlots) & 1, abort_flag)) { record_failure(abort_flag, kSiteMmaS); ok = false; break; }
          }
          const uint32_t s = kc % kKStages;
          if (!mbar_wait_warp(&bars[kBarKFull + s], (kc / kKStages) & 1, abort_flag)) { record_failure(abort_flag, kSiteMmaK); ok = false; break; }
          tc_fence_after();
          const uint32_t sfb = tmem + kColSFB + (kc & 1) * 4;
          tmem_cp_32x128b_x4(sfb, dksf0 + (s * kAtomBytes >> 4), leader);
          const uint64_t bdesc = dk0 + (s * kTileBytes >> 4);
          const uint32_t d = tmem + kColS + b * 128;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {  // K = 32 bytes per MMA
            const uint32_t byte_sel = static_cast<uint32_t>(kk) << 30;
            mma_mxf8f6f4_ss(d, adesc + kk * 2, bdesc + kk * 2, idq[kk], sfa | byte_sel, sfb | byte_sel,
                            kk > 0 ? 1u : 0u, leader);
          }
          mma_commit(&bars[kBarSFull + b], leader);
          mma_commit(&bars[kBarKEmpty + s], leader);
          if (j == ui.nkv - 1) mma_commit(&bars[kBarQEmpty + qs], leader);
          ++kc;
        }
        ++u;
      }
      // Drain: wait until every tcgen05 operation issued by this warp has completed.
      mma_commit(&bars[kBarDrain], leader);
      if (!mbar_wait(&bars[kBarDrain], 0, nullptr)) record_failure(abort_flag, kSiteDrain);
    } else if (warp == 2) {
      // ---------------------------------------------------------------- PV issuer
      // O += P(t) V(t). A warp of its own, so that waiting for the softmax (PReady) never
      // holds back the next QK.
      const uint32_t leader = lane == 0 ? 1u : 0u;
      const uint32_t sb = static_cast<uint32_t>(warp_uniform(static_cast<int>(smem_u32(smem))));
      const uint64_t dv0 = kP8 ? umma_desc(sb + L::v, kTileBytes, 1024, kLayoutSw128)
                               : umma_desc(sb + L::vbf, kTileBytes, 1024, kLayoutSw128);
      const uint64_t dpsf0 = umma_desc(sb + L::p_sf, 0, 128, kLayoutNone);
      const uint64_t dvsf0 = umma_desc(sb + L::v_sf, 0, 128, kLayoutNone);
      uint32_t u = 0, vc = 0, t = 0;  // units, V tiles, tiles
      bool ok = true;
      for (int w = blockIdx.x; w < p.num_units && ok; w += G) {
        const UnitInfo ui = warp_uniform(unit_info(p, sched, w));
        if (ui.nkv == 0) continue;
        for (int j = 0; j < ui.nkv; ++j, ++t) {
          const uint32_t b = t & 1;
          if (!mbar_wait_warp(&bars[kBarPReady + t % kPSlots], (t / kPSlots) & 1, abort_flag)) { record_failure(abort_flag, kSiteMmaP); ok = false; break; }
          if (j == 0 && !mbar_wait_warp(&bars[kBarOEmpty], (u & 1) ^ 1, abort_flag)) { record_failure(abort_flag, kSiteMmaO); ok = false; break; }
          const bool got = kP8 ? mbar_wait_warp(&bars[kBarVFull + vc % kVStages], (vc / kVStages) & 1, abort_flag)
                               : mbar_wait_warp(&bars[kBarVbfFull + vc % kVbfStages], (vc / kVbfStages) & 1, abort_flag);
          if (!got) { record_failure(abort_flag, kSiteMmaV); ok = false; break; }
          tc_fence_after();
          if (kMx) {
            // Scale atoms into TMEM (the copies run in order with the MMAs below): P's from the
            // softmax's shared-memory atom of this slot, V's from the V stage.
            const uint32_t sfp = tmem + kColSFP + (t & 1) * 4;
            const uint32_t sfv = tmem + kColSFV + (vc & 1) * 4;
            tmem_cp_32x128b_x4(sfp, dpsf0 + ((t % kPSlots) * kAtomBytes >> 4), leader);
            tmem_cp_32x128b_x4(sfv, dvsf0 + ((vc % kVStages) * kAtomBytes >> 4), leader);
            const uint32_t p_col = tmem + kColP + (t % kPSlots) * 32;
            const uint64_t bdesc = dv0 + ((vc % kVStages) * kTileBytes >> 4);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {  // keys [32kk, 32kk + 32), scale byte kk
              const uint32_t byte_sel = static_cast<uint32_t>(kk) << 30;
              mma_mxf8f6f4_ts(tmem + kColO, p_col + kk * 8, bdesc + kk * 256, idesc_pv_mx(kk), sfp | byte_sel,
                              sfv | byte_sel, (j > 0 || kk > 0) ? 1u : 0u, leader);
            }
            mma_commit(&bars[kBarVEmpty + vc % kVStages], leader);
          } else if (kFp8PV) {
            const uint32_t p_col = tmem + kColP + (t % kPSlots) * 32;
            const uint64_t bdesc = dv0 + ((vc % kVStages) * kTileBytes >> 4);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)  // keys [32kk, 32kk + 32): 8 columns of 4 E4M3 each
              mma_f8f6f4_ts(tmem + kColO, p_col + kk * 8, bdesc + kk * 256, kIdescPV8,
                            (j > 0 || kk > 0) ? 1u : 0u, leader);
            mma_commit(&bars[kBarVEmpty + vc % kVStages], leader);
          } else {
            const uint32_t p_col = tmem + kColS + b * 128;
            const uint64_t bdesc = dv0 + ((vc % kVbfStages) * kVbfBytes >> 4);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)  // keys [16kk, 16kk + 16): 8 columns of 2 BF16 each
              mma_f16_ts(tmem + kColO, p_col + kk * 8, bdesc + kk * 128, kIdescPV16,
                         (j > 0 || kk > 0) ? 1u : 0u, leader);
            mma_commit(&bars[kBarVbfEmpty + vc % kVbfStages], leader);
          }
          mma_commit(&bars[kBarPVDone + t % kPSlots], leader);
          ++vc;
        }
        if (!ok) break;
        mma_commit(&bars[kBarOFull], leader);  // every PV of this unit is complete
        ++u;
      }
      mma_commit(&bars[kBarDrainPV], leader);
      if (!mbar_wait(&bars[kBarDrainPV], 0, nullptr)) record_failure(abort_flag, kSiteDrain);
    }
  } else if (warp < 12) {
    setmaxnreg_inc<kSoftmaxRegs>();
    // ------------------------------------------------------------------ softmax groups
    // (Block-scaled P has no E4M3 range limit to respect: it takes the bf16 mode's lag.)
    constexpr float kLag = SoftmaxLag<kFp8PV>::lag;
    constexpr float kBias = SoftmaxLag<kFp8PV>::bias;
    uint32_t* p_sf_words = reinterpret_cast<uint32_t*>(smem + L::p_sf);
    const uint32_t grp = static_cast<uint32_t>(warp - 4) >> 2;  // tiles t with t & 1 == grp
    const int quarter = warp & 3;                                // TMEM lane quarter of this warp
    const int row = quarter * 32 + lane;                         // query row within the tile
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    float* my_mref = mref + grp * 128 + row;
    const float* other_mref = mref + (grp ^ 1) * 128 + row;
    // |logit scale|; the sign is folded into the QK MMA. With per-tensor q/k descales it is the
    // same for every unit and is computed once here; kPerUnitDescale reads it per unit.
    const float cscale_all = kPerUnitDescale ? 0.0f
                                             : fabsf((descale_value(p.q_descale, 0, 0) *
                                                      descale_value(p.k_descale, 0, 0)) * kLog2eRsqrtD);
    uint32_t u = 0, t0 = 0;
    bool ok = true;
    for (int w = blockIdx.x; w < p.num_units && ok; w += G) {
      const UnitInfo ui = unit_info(p, sched, w);
      if (ui.nkv == 0) {
        // No keys: an empty sum, LSE = log 0 = -inf and O = 0.
        if (ui.qtile * kTileM + row < ui.q_len) {
          const int64_t tok = ui.q_row0 + row;
          uint4* dst = reinterpret_cast<uint4*>(p.out + (tok * p.heads + ui.h) * 128 + grp * 64);
#pragma unroll
          for (int c = 0; c < 8; ++c) dst[c] = make_uint4(0u, 0u, 0u, 0u);
          if (grp == 0) p.lse[static_cast<int64_t>(ui.h) * p.tq + tok] = -INFINITY;
        }
        continue;
      }
      // (v's descale is read in the epilogue, so that nothing more stays live across the tiles.)
      const float cscale = kPerUnitDescale ? fabsf((descale_value(p.q_descale, ui.seq, ui.h) *
                                                    descale_value(p.k_descale, ui.seq, ui.h)) * kLog2eRsqrtD)
                                           : cscale_all;
      float m_g = -INFINITY;  // reference this group's l is relative to (-inf: no tile yet)
      float l_g = 0.0f;       // this group's sum of p over its tiles (times 2^kBias)
      float lr_g = 0.0f;      // bf16 PV mode: the same sum over the BF16-rounded P
      for (int j = static_cast<int>((t0 ^ grp) & 1); j < ui.nkv; j += 2) {
        const uint32_t t = t0 + j;           // t & 1 == grp
        const uint32_t kt = t >> 1;          // this group's tile ordinal
        if (!mbar_wait_warp(&bars[kBarSFull + grp], kt & 1, abort_flag)) { record_failure(abort_flag, kSiteSoftS); ok = false; break; }
        tc_fence_after();
        float2 sv[64];
        load_row(tmem + lane_addr + kColS + grp * 128, sv);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[kBarSFree + grp]);  // S buffer may be overwritten
        const int key0 = j * kTileN;
        const bool tail = key0 + kTileN > ui.k_len;
        if (tail) mask_keys(sv, key0, ui.k_len);
        // Every tile has a valid key, so the ceiling is finite.
        float gmax[4];  // block-scaled MXFP8 P: the 32-key group maxima of S
        const float c_t = ceilf((kMx ? rowmax128_groups(sv, gmax) : rowmax128(sv)) * cscale);
        // Reference of tile t - 1 (the other group's). It is published after the other
        // group's exponentials of tile t - 1, so this wait also hands the MUFU over from one
        // group to the other: the two groups' exponential phases alternate instead of
        // competing, and each group's load, max and P stores overlap the other's
        // exponentials. Every tile waits, even the first of a unit, which keeps the hand-over
        // (and the tile references) in tile order.
        float m_prev = 0.0f;
        if (t >= 1) {
          if (!mbar_wait_warp(&bars[kBarMRef + (grp ^ 1) * 4 + quarter], ((t - 1) >> 1) & 1, abort_flag)) { record_failure(abort_flag, kSiteSoftRed); ok = false; break; }
          m_prev = *other_mref;
        }
        const float m_t = (j == 0 || c_t > m_prev + kLag) ? c_t : m_prev;
        *my_mref = m_t;
        auto handoff = [&](float dep) {
          __syncwarp();
          if (lane == 0) mbar_arrive_after(&bars[kBarMRef + grp * 4 + quarter], dep);
        };
        float psum;
        uint32_t mx_sfw = 0;  // block-scaled MXFP8 P: this row's four E8M0 scale bytes
        if (kMx) {
          // Group g: the largest p is ex2(gmax * c + nb) (ex2 and the fma are monotonic), which
          // picks 2^e_g (RCEIL); the exponentials then run with bias nb - e_g, giving p * 2^-e_g.
          const float nb = kBias - m_t;
          float nbg[4], gsum[4];
          int eg[4];
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            eg[g] = e8m0_exponent(ex2_approx(fmaf(gmax[g], cscale, nb)), 0);
            nbg[g] = nb - static_cast<float>(eg[g]);
            mx_sfw |= static_cast<uint32_t>(eg[g] + 127) << (8 * g);
          }
          if (tail) exp_row_groups<true>(sv, cscale, nbg, key0, ui.k_len, handoff, gsum);
          else exp_row_groups<false>(sv, cscale, nbg, key0, ui.k_len, handoff, gsum);
          psum = 0.0f;
#pragma unroll
          for (int g = 0; g < 4; ++g)  // sum of the unscaled p: exact powers of two (2^-126 for an empty group)
            psum += gsum[g] * __uint_as_float(static_cast<uint32_t>(max(eg[g], -126) + 127) << 23);
        } else {
          psum = tail ? exp_row<true, kPolyPairs>(sv, cscale, kBias - m_t, key0, ui.k_len, handoff)
                      : exp_row<false, kPolyPairs>(sv, cscale, kBias - m_t, key0, ui.k_len, handoff);
        }
        const float l_scale = exp2_int(m_g - m_t);
        l_g = l_g * l_scale + psum;
        if (!kP8) lr_g *= l_scale;
        m_g = m_t;
        if (kP8) {
          // PV(t - 3) has read the previous P of this slot. (In bf16 PV mode P goes over the S
          // buffer, which QK(t) only overwrote after PV(t - 2) had completed.)
          if (t >= kPSlots) {
            if (!mbar_wait_warp(&bars[kBarPVDone + t % kPSlots], ((t - kPSlots) / kPSlots) & 1, abort_flag)) { record_failure(abort_flag, kSiteSoftPV); ok = false; break; }
            tc_fence_after();
          }
          if (kMx) {
            // MXFP8 P (already p * 2^-e_g from the exponentials, so at most ~448 per group; the
            // conversion below saturates): the row's four scale bytes go to the slot's
            // shared-memory atom (row r at (r % 32) * 16 + (r / 32) * 4).
            p_sf_words[(t % kPSlots) * (kAtomBytes / 4) + (row & 31) * 4 + (row >> 5)] = mx_sfw;
            fence_proxy_async_smem();  // the PV issuer's tcgen05.cp reads the atom
          }
          uint32_t pk[32];
#pragma unroll
          for (int i = 0; i < 32; ++i)
            pk[i] = static_cast<uint32_t>(cvt_e4m3x2(sv[2 * i].x, sv[2 * i].y)) |
                    (static_cast<uint32_t>(cvt_e4m3x2(sv[2 * i + 1].x, sv[2 * i + 1].y)) << 16);
          tmem_st32_sync(tmem + lane_addr + kColP + (t % kPSlots) * 32, pk);
        } else {
          // O is normalised by the sum of the P values the PV product actually uses, so a
          // row dominated by one key gets that V row exactly (the LSE keeps the unrounded sum).
          float2 racc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t pk[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              pk[i] = cvt_bf16x2(sv[32 * h + i].x, sv[32 * h + i].y);
              racc[i & 3] = __fadd2_rn(racc[i & 3], make_float2(__uint_as_float(pk[i] << 16),
                                                               __uint_as_float(pk[i] & 0xFFFF0000u)));
            }
            tmem_st32_sync(tmem + lane_addr + kColS + grp * 128 + h * 32, pk);
          }
          const float2 rs = __fadd2_rn(__fadd2_rn(racc[0], racc[1]), __fadd2_rn(racc[2], racc[3]));
          lr_g += rs.x + rs.y;
        }
        // O holds tiles up to t - 1 relative to m_prev; rescale it when the reference moved
        // (rare; never on a unit's first tile).
        if (j > 0 && __any_sync(0xFFFFFFFFu, m_t != m_prev)) {
          if (!mbar_wait_warp(&bars[kBarPVDone + (t - 1) % kPSlots], ((t - 1) / kPSlots) & 1, abort_flag)) { record_failure(abort_flag, kSiteSoftO); ok = false; break; }
          tc_fence_after();
          const float alpha = exp2_int(m_prev - m_t);
          const float2 a2 = make_float2(alpha, alpha);
          const uint32_t o_addr = tmem + lane_addr + kColO;
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t ro[32];
            tmem_ld32_sync(o_addr + c * 32, ro);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float2 o2 = __fmul2_rn(make_float2(__uint_as_float(ro[2 * i]), __uint_as_float(ro[2 * i + 1])), a2);
              ro[2 * i] = __float_as_uint(o2.x);
              ro[2 * i + 1] = __float_as_uint(o2.y);
            }
            tmem_st32_sync(o_addr + c * 32, ro);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[kBarPReady + t % kPSlots]);
      }
      if (!ok) break;
      t0 += ui.nkv;
      // ---------------------------------------------------------------- epilogue
      // OFull completes once per unit, after the unit's last PV (so after every rescale).
      if (!mbar_wait_warp(&bars[kBarOFull], u & 1, abort_flag)) { record_failure(abort_flag, kSiteSoftPV); ok = false; break; }
      tc_fence_after();
      lsum[grp * 128 + row] = l_g;
      mfin[grp * 128 + row] = m_g;
      if (!kP8) lsumr[grp * 128 + row] = lr_g;
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kBarLReady]);
      if (!mbar_wait_warp(&bars[kBarLReady], u & 1, abort_flag)) { record_failure(abort_flag, kSiteSoftL); ok = false; break; }
      const float m_o = mfin[(grp ^ 1) * 128 + row];
      const float l_o = lsum[(grp ^ 1) * 128 + row];
      const float m_f = fmaxf(m_g, m_o);  // the unit's last reference (references never fall)
      const float s_g = exp2_int(m_g - m_f), s_o = exp2_int(m_o - m_f);
      const float ltot = l_g * s_g + l_o * s_o;
      const float vd = descale_value(p.v_descale, ui.seq, ui.h);
      const float oscale = kP8 ? vd / ltot : vd / (lr_g * s_g + lsumr[(grp ^ 1) * 128 + row] * s_o);
      uint32_t ra[32], rb[32];
      tmem_ld64_sync(tmem + lane_addr + kColO + grp * 64, ra, rb);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kBarOEmpty]);
      if (ui.qtile * kTileM + row < ui.q_len) {
        const int64_t tok = ui.q_row0 + row;
        uint4* dst = reinterpret_cast<uint4*>(p.out + (tok * p.heads + ui.h) * 128 + grp * 64);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint4 v;
          v.x = cvt_bf16x2(__uint_as_float(ra[8 * c + 0]) * oscale, __uint_as_float(ra[8 * c + 1]) * oscale);
          v.y = cvt_bf16x2(__uint_as_float(ra[8 * c + 2]) * oscale, __uint_as_float(ra[8 * c + 3]) * oscale);
          v.z = cvt_bf16x2(__uint_as_float(ra[8 * c + 4]) * oscale, __uint_as_float(ra[8 * c + 5]) * oscale);
          v.w = cvt_bf16x2(__uint_as_float(ra[8 * c + 6]) * oscale, __uint_as_float(ra[8 * c + 7]) * oscale);
          dst[c] = v;
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint4 v;
          v.x = cvt_bf16x2(__uint_as_float(rb[8 * c + 0]) * oscale, __uint_as_float(rb[8 * c + 1]) * oscale);
          v.y = cvt_bf16x2(__uint_as_float(rb[8 * c + 2]) * oscale, __uint_as_float(rb[8 * c + 3]) * oscale);
          v.z = cvt_bf16x2(__uint_as_float(rb[8 * c + 4]) * oscale, __uint_as_float(rb[8 * c + 5]) * oscale);
          v.w = cvt_bf16x2(__uint_as_float(rb[8 * c + 6]) * oscale, __uint_as_float(rb[8 * c + 7]) * oscale);
          dst[4 + c] = v;
        }
        if (grp == 0) p.lse[static_cast<int64_t>(ui.h) * p.tq + tok] = (m_f - kBias + lg2_approx(ltot)) * kLn2;
      }
      ++u;
    }
  } else {
    setmaxnreg_dec<kOtherRegs>();
    if (kPv == kPvBf16Mx) {
      // ---------------------------------------------------------------- V converter (bf16 PV)
      const int t = threadIdx.x - 12 * 32;  // key row of the V tile, 0..127
      const uint32_t sw = static_cast<uint32_t>(t & 7);
      uint32_t vc = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < p.num_units && ok; w += G) {
        const UnitInfo ui = unit_info(p, sched, w);
        for (int j = 0; j < ui.nkv; ++j) {
          const uint32_t s = vc % kVStages, ph = (vc / kVStages) & 1;
          const uint32_t sb = vc % kVbfStages, phb = (vc / kVbfStages) & 1;
          if (!mbar_wait_warp(&bars[kBarVFull + s], ph, abort_flag)) { record_failure(abort_flag, kSiteConvV); ok = false; break; }
          if (!mbar_wait_warp(&bars[kBarVbfEmpty + sb], phb ^ 1, abort_flag)) { record_failure(abort_flag, kSiteConvE); ok = false; break; }
          const uint8_t* src = smem + L::v + s * kTileBytes + t * 128;
          const uint32_t sfw = reinterpret_cast<const uint32_t*>(smem + L::v_sf + s * kAtomBytes)[(t & 31) * 4 + (t >> 5)];
          uint8_t* dst = smem + L::vbf + sb * kVbfBytes + t * 128;
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
            // bf16 chunks 2c and 2c+1 (8 elements each) of the MN-major SW128 layout:
            // atom a = chunk / 8 holds head_dim [64a, 64a + 64); rows are keys.
#pragma unroll
            for (int hc = 0; hc < 2; ++hc) {
              const uint32_t chunk = 2 * c + hc;
              const uint32_t atom = chunk >> 3, cc = chunk & 7;
              *reinterpret_cast<uint4*>(dst + atom * kTileBytes + ((cc ^ sw) << 4)) =
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
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(*tmem_slot, kTmemCols);  // the address the allocation returned
  }
}

}  // namespace lpfa
