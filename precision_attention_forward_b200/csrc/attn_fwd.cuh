// attn_fwd.cuh -- definitions shared by the attention forward kernel (attn_fwd_pp.cuh): launch
// shape and register split, descales, kernel parameters, UMMA descriptors, and the softmax row
// helpers (TMEM row loads, key masking, row maxima, exponentials).
//
// The forward computes, per (sequence, head), O = softmax(Q K^T * qd * kd / sqrt(128)) V * vd and
// the natural-log LSE for noncausal head_dim 128 over packed variable-length sequences (LP-FA4
// README, "MXFP8 forward and backward"); absent descales are the literal 1.0f on the same code
// path (vLLM #63232, "Claims").
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
constexpr uint32_t kTileBytes = 128 * 128;     // 128 rows x 128 fp8
constexpr uint32_t kAtomBytes = 512;

constexpr uint32_t kTmemCols = 512;

// log2(e) / sqrt(128) rounded to fp32: logits in log2 units per unit of Q.K.
constexpr float kLog2eRsqrtD = 0.12751743082459868f;
constexpr float kLn2 = 0.69314718055994531f;


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
  int shared_q;             // 1: one query sequence shared by num_seqs key/value sequences; output
                            // block i (rows i * Lq ..) belongs to key/value sequence i
};

// Work order: up to this many sequences are ordered longest first (by key tiles) in shared
// memory at the start of the kernel; beyond it units keep the plain head-major order.
#ifndef LPFA_MAX_SORT_SEQS
#define LPFA_MAX_SORT_SEQS 256
#endif
constexpr int kMaxSortSeqs = LPFA_MAX_SORT_SEQS;


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

// Block-scaled MXFP8 P: p = 2^(s c + nb) in place, group g (pairs [16g, 16g + 16)) with its own
// bias nbg[g] = nb - e_g, so the exponentials come out already scaled by the group's 2^-e_g (an
// integer shift of the exponent). Masked keys (tail tiles) become exactly 0. gsum[g] receives the
// sum of the group's scaled p.
template <bool kTail>
__device__ __forceinline__ void exp_row_groups(float2 (&s)[64], float c, const float (&nbg)[4], int key0, int klen,
                                               float (&gsum)[4]) {
  const float2 c2 = make_float2(c, c);
#pragma unroll
  for (int i = 0; i < 64; ++i) s[i] = __ffma2_rn(s[i], c2, make_float2(nbg[i >> 4], nbg[i >> 4]));
#pragma unroll
  for (int i = 0; i < 64; ++i) s[i] = exp2_mufu2(s[i]);
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


__device__ __forceinline__ int find_prefix(const int32_t* prefix, int n, int g) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(prefix + mid) <= g) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ int find_prefix_smem(const int* prefix, int n, int g) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= g) lo = mid; else hi = mid - 1;
  }
  return lo;
}



// Warp-uniform copies of values that every lane of a warp computes identically. Results of
// warp votes and reductions live in uniform registers, which lets the compiler keep the
// producer and MMA loops (trip counts, stage indices, descriptors) on the uniform datapath;
// otherwise every tcgen05.mma operand would need a per-instruction register conversion.
__device__ __forceinline__ int warp_uniform(int x) {
  return static_cast<int>(__reduce_max_sync(0xFFFFFFFFu, static_cast<unsigned>(x)));
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

// How far (log2 units) a row's logits may exceed its reference before the reference, l and O
// move, and the power of two P is computed with, for bf16 P and block-scaled MXFP8 P: bf16 P
// keeps its 8-bit mantissa at any scale and block-scaled P absorbs any power of two in its E8M0
// scale, so both may lag 8 binades. (fp8 P, bounded by the E4M3 range, has its own.)
constexpr float kLagWide = 8.0f;
constexpr float kBiasWide = 0.0f;


}  // namespace lpfa
