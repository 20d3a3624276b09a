// attn_bwd.cuh -- MXFP8 attention backward for sm_100a (noncausal, head_dim 128, varlen).
//
// Computes, per (sequence, head), the gradients of O = softmax(Q K^T * c) V * vd (c = qd * kd /
// sqrt(128)) with respect to the dequantized Q, K, V, from O, dO and the forward's LSE (LP-FA4
// README, "MXFP8 forward and backward": mxfp8_flash_attn_varlen_backward returns dQ in BF16 and dK,
// dV as BF16 or, with output_mxfp8_dkv, as E4M3 payloads with one E8M0 scale per 32 elements):
//
//   P = exp(S - LSE),  dV = vd P^T dO,  dP = vd dO V^T,  D = rowsum(dO * O),
//   dS = P * (dP - D),  dQ = c dS K,  dK = c dS^T Q.
//
// Three kernels, no scratch memory:
//   attn_bwd_d_kernel     D for every (token, head), written as fp32 into the dQ output buffer,
//                         which nothing else reads or writes until the dQ kernel overwrites it.
//   attn_bwd_dkdv_kernel  one CTA per 128-key tile of a (sequence, head): over the sequence's
//                         query tiles it recomputes S^T = K Q^T and dP^T = V dO^T, forms P^T and
//                         dS^T (one thread per key row) and accumulates dV += P^T dO and
//                         dK += dS^T Q in tensor memory.
//   attn_bwd_dq_kernel    one CTA per 128-row query tile: over the key tiles it recomputes S and
//                         dP, forms dS (one thread per query row) and accumulates dQ += dS K; it
//                         computes its own tile's D from dO and O.
// Each CTA dequantizes its MXFP8 tiles to BF16 in shared memory (exact: E4M3 * 2^e is a BF16
// value) and runs BF16 tcgen05 MMAs, so no scale factors are needed in tensor memory.
//
// Warp roles (288 threads): warps 0-3 compute (one tile row per thread: the TMEM reads and writes
// of the row updates), warp 4 issues the MMAs, warps 5-8 load. The loaders fill a two-stage ring
// of the streamed tiles (Q, dO, D, LSE in the dK/dV kernel; K, V in the dQ kernel) with
// coalesced 16-byte loads, converting as they store. Per step the S and dP MMAs run with N = 128
// (a 64-column split measured 2-3x slower per flop on the tensor core); the accumulating MMAs
// follow the row updates 32 columns at a time, and the next step's S/dP MMAs are issued as soon
// as their TMEM columns are free.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "ptx.cuh"

namespace lpfa {

constexpr int kBwdThreads = 288;                 // warps 0-3 compute, warp 4 MMA issue, warps 5-8 load
constexpr int kBwdIssueWarp = 4;
constexpr int kBwdLoadWarp0 = 5;
constexpr uint32_t kBfTile = 128 * 128 * 2;      // a 128 x 128 BF16 tile in shared memory
constexpr uint32_t kBfAtom = 128 * 128;          // one 64-column half of it (SW128 atom column)

struct BwdParams {
  const uint8_t* q;         // (Tq, H, 128) E4M3, head_dim-orientation scales q_sf
  const uint8_t* q_sf;
  const uint8_t* k;
  const uint8_t* k_sf;
  const uint8_t* v;
  const uint8_t* v_sf;
  const __nv_bfloat16* o;   // (Tq, H, 128)
  const __nv_bfloat16* dout;
  const float* lse;         // (H, Tq)
  const int32_t* cu_q;
  const int32_t* so_q;
  const int32_t* cu_k;
  const int32_t* so_k;
  Descale q_descale, k_descale, v_descale;
  __nv_bfloat16* dq;        // (Tq, H, 128)
  void* dk;                 // (Tk, H, 128): BF16, or E4M3 payload with dk_sf
  void* dv;
  uint8_t* dk_sf;           // MXFP8 output scale storage (under meta_k) or nullptr
  uint8_t* dv_sf;
  int num_seqs;
  int heads;
  int tq;
  int total_q_tiles;
  int total_k_tiles;
  int mxfp8_dkv;
  int debug_stall;          // test hook: > 0 makes the dK/dV kernel's MMA warp wait on a phase that never comes
};

// Byte offset of element chunk (8 BF16) cc of row r in a 128-row BF16 tile stored as two
// 128 x 64 SW128 atoms (columns [0, 64) and [64, 128)): the layout TMA's 128-byte swizzle
// produces and the MMA reads, K-major (rows are M or N) or MN-major (rows are K) alike.
__device__ __forceinline__ uint32_t bf_tile_offset(int r, int chunk) {
  const uint32_t atom = static_cast<uint32_t>(chunk) >> 3, cc = static_cast<uint32_t>(chunk) & 7u;
  return atom * kBfAtom + static_cast<uint32_t>(r) * 128u + ((cc ^ (static_cast<uint32_t>(r) & 7u)) << 4);
}

// 16 E4M3 codes (one 16-byte piece of a row) times 2^e as 16 BF16 values (two 8-value chunks).
__device__ __forceinline__ void mx16_to_bf(const uint4 raw, uint32_t sbyte, uint4& lo, uint4& hi) {
  const int e = static_cast<int>(sbyte) - 127;
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
  lo = make_uint4(outw[0], outw[1], outw[2], outw[3]);
  hi = make_uint4(outw[4], outw[5], outw[6], outw[7]);
}

// dot of two pieces of 8 BF16 values, in fp32.
__device__ __forceinline__ float bf8_dot(const uint4 x, const uint4 y) {
  const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
  float acc = 0.0f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    acc = fmaf(__uint_as_float(xs[i] << 16), __uint_as_float(ys[i] << 16), acc);
    acc = fmaf(__uint_as_float(xs[i] & 0xFFFF0000u), __uint_as_float(ys[i] & 0xFFFF0000u), acc);
  }
  return acc;
}

// BF16 x BF16 -> F32, M = 128, N = n; a_mn / b_mn: operand is MN-major (else K-major).
__device__ __forceinline__ constexpr uint32_t idesc_bf16(bool a_mn, bool b_mn, uint32_t n = 128) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (a_mn ? (1u << 15) : 0u) | (b_mn ? (1u << 16) : 0u) |
         ((n >> 3) << 17) | (8u << 24);
}

// Descriptor of K step kk (16 elements) of a BF16 tile: K-major operands step 32 bytes inside an
// SW128 atom row and move to the second atom after 4 steps; MN-major operands step 16 rows.
__device__ __forceinline__ uint64_t bf_kmajor_step(uint64_t base, int kk) {
  return base + static_cast<uint64_t>((kk >> 2) * (kBfAtom >> 4) + (kk & 3) * 2);
}
__device__ __forceinline__ uint64_t bf_mnmajor_step(uint64_t base, int kk) {
  return base + static_cast<uint64_t>(kk * (16 * 128 >> 4));
}

constexpr float kBwdLog2e = 1.4426950408889634f;
constexpr float kBwdRsqrtD = 0.08838834764831845f;  // 1 / sqrt(128)

// Shared memory of the two tile kernels (offsets from the 1024-aligned base):
//   [0, 64K)        the resident pair: K, V (dK/dV kernel) or Q, dO (dQ kernel), BF16 tiles
//   [64K, 192K)     two stages of the streamed pair: Q, dO or K, V
//   [192K, +2K)     per stage: LSE (log2 units) and D, 128 floats each (dK/dV kernel); stage 0
//                   holds the resident query tile's in the dQ kernel
//   then            barriers, the TMEM slot, the abort flag
constexpr uint32_t kBwdOffStage = 2 * kBfTile;
constexpr uint32_t kBwdStageBytes = 2 * kBfTile;
constexpr uint32_t kBwdOffVec = kBwdOffStage + 2 * kBwdStageBytes;
constexpr uint32_t kBwdOffBar = kBwdOffVec + 2 * 2 * 128 * 4;
constexpr uint32_t kBwdNumBars = 13;
constexpr uint32_t kBwdSmem = kBwdOffBar + kBwdNumBars * 8 + 16 + 1024;
static_assert(kBwdSmem <= 227 * 1024, "backward shared memory over the per-CTA limit");

// Barrier indices. Arrival counts: the loaders' 128 threads (resident, stage full), the compute
// warps' 128 threads (chunk ready), one tcgen05.commit (the others).
constexpr int kBbResident = 0;   // resident pair (and the dQ kernel's D, LSE) in shared memory
constexpr int kBbFull = 1;       // + stage: streamed tile in shared memory
constexpr int kBbEmpty = 3;      // + stage: the last MMA that reads the stage is done
constexpr int kBbSFull = 5;      // S and dP of the step in TMEM
constexpr int kBbChunk = 6;      // + chunk (4): the chunk's P and dS in TMEM (compute threads)
constexpr int kBbRFree = 10;     // the step's accumulating MMAs are done
constexpr int kBbDrain = 12;     // every MMA the issue warp issued is done (before teardown)

struct BwdSmem {
  uint8_t* base;
  __device__ uint8_t* res0() const { return base; }
  __device__ uint8_t* res1() const { return base + kBfTile; }
  __device__ uint8_t* st0(int s) const { return base + kBwdOffStage + s * kBwdStageBytes; }
  __device__ uint8_t* st1(int s) const { return base + kBwdOffStage + s * kBwdStageBytes + kBfTile; }
  __device__ float* lse(int s) const { return reinterpret_cast<float*>(base + kBwdOffVec + s * 1024); }
  __device__ float* dvec(int s) const { return reinterpret_cast<float*>(base + kBwdOffVec + s * 1024 + 512); }
  __device__ uint64_t* bar(int i) const { return reinterpret_cast<uint64_t*>(base + kBwdOffBar) + i; }
  __device__ uint32_t* tslot() const { return reinterpret_cast<uint32_t*>(base + kBwdOffBar + kBwdNumBars * 8); }
  __device__ int* abort_flag() const { return reinterpret_cast<int*>(base + kBwdOffBar + kBwdNumBars * 8 + 8); }
};

// A 128 x 128 block of fp32 results in TMEM, rows on lanes, written out as BF16 rows (rows < n),
// or as MXFP8 (head_dim orientation, RCEIL: 32 columns = one block) with its scale atom.
__device__ __forceinline__ void bwd_store_rows(uint32_t taddr, float scale, int r, int n, int64_t out_row,
                                               void* out, uint8_t* atom, bool mx) {
#pragma unroll 1
  for (int cb = 0; cb < 4; ++cb) {
    uint32_t x[32];
    tmem_ld32_sync(taddr + cb * 32, x);
    float v[32];
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      v[i] = __uint_as_float(x[i]) * scale;
      amax = fmaxf(amax, fabsf(v[i]));
    }
    if (!mx) {
      if (r < n) {
        uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(out) + out_row * 128 + cb * 32);
#pragma unroll
        for (int c = 0; c < 4; ++c)
          dst[c] = make_uint4(cvt_bf16x2(v[8 * c], v[8 * c + 1]), cvt_bf16x2(v[8 * c + 2], v[8 * c + 3]),
                              cvt_bf16x2(v[8 * c + 4], v[8 * c + 5]), cvt_bf16x2(v[8 * c + 6], v[8 * c + 7]));
      }
    } else {
      const int e = e8m0_exponent(amax, 0);
      const float inv = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);
      if (r < n) {
        uint4* dst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(out) + out_row * 128 + cb * 32);
        uint32_t w[8];
#pragma unroll
        for (int k = 0; k < 8; ++k)
          w[k] = static_cast<uint32_t>(cvt_e4m3x2(v[4 * k] * inv, v[4 * k + 1] * inv)) |
                 (static_cast<uint32_t>(cvt_e4m3x2(v[4 * k + 2] * inv, v[4 * k + 3] * inv)) << 16);
        dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
        dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
      }
      atom[(r & 31) * 16 + (r >> 5) * 4 + cb] = r < n ? static_cast<uint8_t>(e + 127) : uint8_t{0x7F};
    }
  }
}

// D = rowsum(dO * O) for every (token, head), as fp32 at dbuf[h * Tq + token] (the layout of
// LSE). 16 lanes per row, 8 values per lane; a warp covers two consecutive rows.
__global__ void __launch_bounds__(256) attn_bwd_d_kernel(const BwdParams p) {
  float* dbuf = reinterpret_cast<float*>(p.dq);
  const int64_t rows = static_cast<int64_t>(p.tq) * p.heads;
  const int lane = threadIdx.x & 31;
  const int64_t warp_step = static_cast<int64_t>(gridDim.x) * (256 / 32) * 2;
  for (int64_t wr = (static_cast<int64_t>(blockIdx.x) * (256 / 32) + (threadIdx.x >> 5)) * 2; wr < rows;
       wr += warp_step) {
    const int64_t rr = wr + (lane >> 4);
    const bool valid = rr < rows;
    uint4 a = make_uint4(0u, 0u, 0u, 0u), b = a;
    if (valid) {
      a = __ldg(reinterpret_cast<const uint4*>(p.dout + rr * 128) + (lane & 15));
      b = __ldg(reinterpret_cast<const uint4*>(p.o + rr * 128) + (lane & 15));
    }
    float d = bf8_dot(a, b);
    d += __shfl_xor_sync(0xFFFFFFFFu, d, 8);
    d += __shfl_xor_sync(0xFFFFFFFFu, d, 4);
    d += __shfl_xor_sync(0xFFFFFFFFu, d, 2);
    d += __shfl_xor_sync(0xFFFFFFFFu, d, 1);
    if (valid && (lane & 15) == 0) {
      const int64_t tok = rr / p.heads;
      const int64_t h = rr - tok * p.heads;
      dbuf[h * p.tq + tok] = d;
    }
  }
}

// ---------------------------------------------------------------------------------------------
// Loaders (warps 5-8; loader warp lw fills rows [32 lw, 32 lw + 32) of a 128-row tile). Every
// load of a tile is issued before the first store, one 16-byte piece per lane; rows >= n are
// written as zeros.
// ---------------------------------------------------------------------------------------------

// A query tile of head h from token tok0 (n rows): Q dequantized to BF16 with its scale atom sf,
// dO copied, LSE in log2 units (+inf past the end, so that p = 0 there) and D, read from the D
// kernel's output (kDFromBuffer) or computed here from dO and O (lanes of a row reduce by
// shuffles).
template <bool kDFromBuffer>
__device__ __forceinline__ void bwd_load_q_tile(const BwdParams& p, int64_t tok0, const uint8_t* sf, int h, int n,
                                                uint8_t* sQ, uint8_t* sDO, float* sD, float* sLse, int lw,
                                                int lane) {
  const int rb = 32 * lw;
  uint4 qv[8];
  uint32_t qs[8];
#pragma unroll
  for (int it = 0; it < 8; ++it) {  // Q: 4 rows per step, 8 lanes x 16 codes per row
    const int r = rb + 4 * it + (lane >> 3);
    qv[it] = make_uint4(0u, 0u, 0u, 0u);
    qs[it] = 0x7F7F7F7Fu;
    if (r < n) {
      qv[it] = __ldg(reinterpret_cast<const uint4*>(p.q + ((tok0 + r) * p.heads + h) * 128) + (lane & 7));
      qs[it] = __ldg(reinterpret_cast<const uint32_t*>(sf) + (r & 31) * 4 + (r >> 5));
    }
  }
  uint4 dv[16], ov[kDFromBuffer ? 1 : 16];
#pragma unroll
  for (int it = 0; it < 16; ++it) {  // dO (and O): 2 rows per step, 16 lanes x 8 values per row
    const int r = rb + 2 * it + (lane >> 4);
    dv[it] = make_uint4(0u, 0u, 0u, 0u);
    if constexpr (!kDFromBuffer) ov[it] = dv[it];
    if (r < n) {
      const int64_t off = ((tok0 + r) * p.heads + h) * 128;
      dv[it] = __ldg(reinterpret_cast<const uint4*>(p.dout + off) + (lane & 15));
      if constexpr (!kDFromBuffer) ov[it] = __ldg(reinterpret_cast<const uint4*>(p.o + off) + (lane & 15));
    }
  }
  const int rl = rb + lane;
  const int64_t vi = static_cast<int64_t>(h) * p.tq + tok0 + rl;
  const float lse2 = rl < n ? __ldg(p.lse + vi) * kBwdLog2e : INFINITY;
  float dval = 0.0f;
  if constexpr (kDFromBuffer) {
    if (rl < n) dval = __ldg(reinterpret_cast<const float*>(p.dq) + vi);
  }
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int r = rb + 4 * it + (lane >> 3), c = lane & 7;  // codes [16c, 16c + 16): block c / 2
    uint4 lo, hi;
    mx16_to_bf(qv[it], (qs[it] >> (8 * (c >> 1))) & 0xFFu, lo, hi);
    *reinterpret_cast<uint4*>(sQ + bf_tile_offset(r, 2 * c)) = lo;
    *reinterpret_cast<uint4*>(sQ + bf_tile_offset(r, 2 * c + 1)) = hi;
  }
#pragma unroll
  for (int it = 0; it < 16; ++it) {
    const int r = rb + 2 * it + (lane >> 4), c = lane & 15;
    *reinterpret_cast<uint4*>(sDO + bf_tile_offset(r, c)) = dv[it];
    if constexpr (!kDFromBuffer) {
      float d = bf8_dot(dv[it], ov[it]);
      d += __shfl_xor_sync(0xFFFFFFFFu, d, 8);
      d += __shfl_xor_sync(0xFFFFFFFFu, d, 4);
      d += __shfl_xor_sync(0xFFFFFFFFu, d, 2);
      d += __shfl_xor_sync(0xFFFFFFFFu, d, 1);
      if (c == 0) sD[r] = d;
    }
  }
  if constexpr (kDFromBuffer) sD[rl] = dval;
  sLse[rl] = lse2;
}

// A key tile of head h from token tok0 (n rows): K and V dequantized to BF16 with the tile's scale
// atoms at byte offset sf_off of k_sf and v_sf.
__device__ __forceinline__ void bwd_load_kv_tile(const BwdParams& p, int64_t tok0, int64_t sf_off, int h, int n,
                                                 uint8_t* sK, uint8_t* sV, int lw, int lane) {
  const int rb = 32 * lw;
  uint4 kv[8], vv[8];
  uint32_t ks[8], vs[8];
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int r = rb + 4 * it + (lane >> 3);
    kv[it] = make_uint4(0u, 0u, 0u, 0u);
    vv[it] = kv[it];
    ks[it] = vs[it] = 0x7F7F7F7Fu;
    if (r < n) {
      const int64_t off = ((tok0 + r) * p.heads + h) * 128;
      const int wi = (r & 31) * 4 + (r >> 5);
      kv[it] = __ldg(reinterpret_cast<const uint4*>(p.k + off) + (lane & 7));
      vv[it] = __ldg(reinterpret_cast<const uint4*>(p.v + off) + (lane & 7));
      ks[it] = __ldg(reinterpret_cast<const uint32_t*>(p.k_sf + sf_off) + wi);
      vs[it] = __ldg(reinterpret_cast<const uint32_t*>(p.v_sf + sf_off) + wi);
    }
  }
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int r = rb + 4 * it + (lane >> 3), c = lane & 7;
    uint4 lo, hi;
    mx16_to_bf(kv[it], (ks[it] >> (8 * (c >> 1))) & 0xFFu, lo, hi);
    *reinterpret_cast<uint4*>(sK + bf_tile_offset(r, 2 * c)) = lo;
    *reinterpret_cast<uint4*>(sK + bf_tile_offset(r, 2 * c + 1)) = hi;
    mx16_to_bf(vv[it], (vs[it] >> (8 * (c >> 1))) & 0xFFu, lo, hi);
    *reinterpret_cast<uint4*>(sV + bf_tile_offset(r, 2 * c)) = lo;
    *reinterpret_cast<uint4*>(sV + bf_tile_offset(r, 2 * c + 1)) = hi;
  }
}

// Barrier setup and TMEM allocation shared by both tile kernels; returns the TMEM base address.
__device__ __forceinline__ uint32_t bwd_setup(const BwdSmem& sm, int tid, int warp) {
  if (tid == 0) {
    for (int b = 0; b < static_cast<int>(kBwdNumBars); ++b) {
      const bool threads = b == kBbResident || b == kBbFull || b == kBbFull + 1 || (b >= kBbChunk && b < kBbChunk + 4);
      mbar_init(sm.bar(b), threads ? 128u : 1u);
    }
    *sm.abort_flag() = 0;
    mbar_fence_init();
  }
  if (warp == 0) tmem_alloc(sm.tslot(), 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  return *sm.tslot();
}

__device__ __forceinline__ void bwd_report(const BwdSmem& sm, int site) {
  *reinterpret_cast<volatile int*>(sm.abort_flag()) = 1;
  if (atomicCAS(&g_lpfa_status[0], 0, 4 /* LPFA_ERR_TIMEOUT */) == 0) atomicExch(&g_lpfa_status[1], site);
}

// Issue warp, on both the normal and the abort exit: every tcgen05 operation it issued completes
// before the CTA reaches its teardown (MMAs still reading shared memory or writing TMEM when
// TMEM is freed would be undefined). The wait is bounded and outlasts an abort; a drain that
// runs out is recorded as site 206.
__device__ __forceinline__ void bwd_drain(const BwdSmem& sm, int lane) {
  mma_commit(sm.bar(kBbDrain), lane == 0 ? 1u : 0u);
  if (!mbar_wait_warp(sm.bar(kBbDrain), 0, nullptr) && lane == 0) bwd_report(sm, 206);
}

// ---------------------------------------------------------------------------------------------
// The pipeline shared by both tile kernels. kDkDv: the dK/dV kernel (resident K, V are the A
// operands of S^T and dP^T; the streamed Q, dO the B operands), else the dQ kernel (resident Q,
// dO; streamed K, V). Step i streams tile i. TMEM columns:
//   0-127      S (fp32, 128 columns: queries in the dK/dV kernel, keys in the dQ kernel); the
//              dK/dV kernel writes P^T as BF16 over 0-63
//   128-255    dP (fp32); the dK/dV kernel writes dS^T as BF16 over 128-191
//   256-383    dV (dK/dV kernel) or dQ (dQ kernel), fp32 accumulators
//   384-511    dK (dK/dV kernel); the dQ kernel writes dS as BF16 over 384-447, apart from S and
//              dP, so that the next step's S/dP MMAs only wait for the row updates to read them
// The row updates go 32 columns at a time; each chunk's accumulating MMAs are issued as soon as
// the chunk is in TMEM, behind the row updates of the next one.
// ---------------------------------------------------------------------------------------------

// MMA issue (warp 4): S/dP of step 0; then per step i the accumulating MMAs chunk by chunk, and
// S/dP of step i + 1 once region 0-255 is free (dK/dV kernel: the accumulating MMAs that read
// P^T and dS^T there are done; dQ kernel: the row updates have read S and dP). Returns false
// when a wait ran out.
template <bool kDkDv>
__device__ __forceinline__ bool bwd_issue(const BwdSmem& sm, uint32_t tm, int n, int lane,
                                          const volatile int* abort_flag) {
  const uint32_t leader = lane == 0 ? 1u : 0u;
  const uint32_t sb = smem_u32(sm.base);
  const uint64_t a1 = umma_desc(sb, 16, 1024, kLayoutSw128);            // K, or Q
  const uint64_t a2 = umma_desc(sb + kBfTile, 16, 1024, kLayoutSw128);  // V, or dO
  constexpr uint32_t idS = idesc_bf16(false, false), idM = idesc_bf16(false, true);
  auto mma_s = [&](int i) {  // S (or S^T) and dP (or dP^T) of step i, N = 128
    const uint32_t st = sb + kBwdOffStage + (i & 1) * kBwdStageBytes;
    const uint64_t b1 = umma_desc(st, 16, 1024, kLayoutSw128);
    const uint64_t b2 = umma_desc(st + kBfTile, 16, 1024, kLayoutSw128);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
      mma_f16_ss(tm, bf_kmajor_step(a1, kk), bf_kmajor_step(b1, kk), idS, kk > 0 ? 1u : 0u, leader);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
      mma_f16_ss(tm + 128, bf_kmajor_step(a2, kk), bf_kmajor_step(b2, kk), idS, kk > 0 ? 1u : 0u, leader);
    mma_commit(sm.bar(kBbSFull), leader);
  };
  if (!mbar_wait_warp(sm.bar(kBbResident), 0, abort_flag)) return false;
  if (n == 0) return true;
  if (!mbar_wait_warp(sm.bar(kBbFull), 0, abort_flag)) return false;
  tc_fence_after();
  mma_s(0);
#pragma unroll 1
  for (int i = 0; i < n; ++i) {
    const int s = i & 1;
    const uint32_t ph = static_cast<uint32_t>(i & 1);
    const uint32_t st = sb + kBwdOffStage + s * kBwdStageBytes;
    const uint64_t m0 = umma_desc(st, kBfAtom, 1024, kLayoutSw128);            // Q, or K (MN-major)
    const uint64_t m1 = umma_desc(st + kBfTile, kBfAtom, 1024, kLayoutSw128);  // dO
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      if (!mbar_wait_warp(sm.bar(kBbChunk + c), ph, abort_flag)) return false;
      tc_fence_after();
#pragma unroll
      for (int kk = 2 * c; kk < 2 * c + 2; ++kk) {
        const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
        if constexpr (kDkDv) {
          mma_f16_ts(tm + 256, tm + 8 * kk, bf_mnmajor_step(m1, kk), idM, acc, leader);        // dV/vd += P^T dO
          mma_f16_ts(tm + 384, tm + 128 + 8 * kk, bf_mnmajor_step(m0, kk), idM, acc, leader);  // dK/c += dS^T Q
        } else {
          mma_f16_ts(tm + 256, tm + 384 + 8 * kk, bf_mnmajor_step(m0, kk), idM, acc, leader);  // dQ/c += dS K
        }
      }
    }
    mma_commit(sm.bar(kBbRFree), leader);
    mma_commit(sm.bar(kBbEmpty + s), leader);  // the last MMA reading stage s
    if (i + 1 < n) {
      if (!mbar_wait_warp(sm.bar(kBbFull + (s ^ 1)), ((i + 1) >> 1) & 1, abort_flag)) return false;
      if (kDkDv && !mbar_wait_warp(sm.bar(kBbRFree), ph, abort_flag)) return false;
      tc_fence_after();
      mma_s(i + 1);
    }
  }
  return true;
}

// Row updates (warps 0-3, thread r = TMEM lane r): per step, 32 columns at a time,
// P = exp2(S c2 - LSE) and dS = P (vd dP - D) from TMEM back to TMEM as BF16. dK/dV kernel: rows
// are keys, columns queries (LSE and D per column, from the stage); dQ kernel: rows are queries
// (LSE and D per row), columns keys, the last tile's columns past last_cols masked. Ends when
// every MMA is done.
template <bool kDkDv>
__device__ __forceinline__ bool bwd_compute(const BwdSmem& sm, uint32_t tm, int n, int warp, int lane, float c2,
                                            float vd, int last_cols, const volatile int* abort_flag) {
  const int r = warp * 32 + lane;
  const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
  const uint32_t trow = tm + lane_addr;
  if (!mbar_wait_warp(sm.bar(kBbResident), 0, abort_flag)) return false;
  float d_r = 0.0f, lse2 = 0.0f;
  if constexpr (!kDkDv) {
    d_r = sm.dvec(0)[r];
    lse2 = sm.lse(0)[r];  // +inf past the sequence: p = 0
  }
#pragma unroll 1
  for (int i = 0; i < n; ++i) {
    const int s = i & 1;
    // The stage's LSE and D (dK/dV kernel) are read directly from shared memory.
    if (kDkDv && !mbar_wait_warp(sm.bar(kBbFull + s), (i >> 1) & 1, abort_flag)) return false;
    if (!mbar_wait_warp(sm.bar(kBbSFull), i & 1, abort_flag)) return false;
    // dQ kernel: the previous step's dQ MMAs read dS from the columns this step's dS overwrites.
    if (!kDkDv && i > 0 && !mbar_wait_warp(sm.bar(kBbRFree), (i - 1) & 1, abort_flag)) return false;
    tc_fence_after();
    const int cols = (!kDkDv && i == n - 1) ? last_cols : 128;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      uint32_t sv[32], dv[32];
      tmem_ld32x2_sync(trow + 32 * c, trow + 128 + 32 * c, sv, dv);
      uint32_t dw[16];
      if constexpr (kDkDv) {
        const float* L = sm.lse(s) + 32 * c;
        const float* D = sm.dvec(s) + 32 * c;
        uint32_t pw[16];
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const float4 l4 = *reinterpret_cast<const float4*>(L + e);
          const float4 d4 = *reinterpret_cast<const float4*>(D + e);
          const float p0 = ex2_approx(fmaf(__uint_as_float(sv[e]), c2, -l4.x));
          const float p1 = ex2_approx(fmaf(__uint_as_float(sv[e + 1]), c2, -l4.y));
          const float p2 = ex2_approx(fmaf(__uint_as_float(sv[e + 2]), c2, -l4.z));
          const float p3 = ex2_approx(fmaf(__uint_as_float(sv[e + 3]), c2, -l4.w));
          pw[e / 2] = cvt_bf16x2(p0, p1);
          pw[e / 2 + 1] = cvt_bf16x2(p2, p3);
          dw[e / 2] = cvt_bf16x2(p0 * fmaf(vd, __uint_as_float(dv[e]), -d4.x),
                                 p1 * fmaf(vd, __uint_as_float(dv[e + 1]), -d4.y));
          dw[e / 2 + 1] = cvt_bf16x2(p2 * fmaf(vd, __uint_as_float(dv[e + 2]), -d4.z),
                                     p3 * fmaf(vd, __uint_as_float(dv[e + 3]), -d4.w));
        }
        // Over columns already read: chunk c writes [16 c, 16 c + 16) of S^T and of dP^T.
        tmem_st16(trow + 16 * c, pw);
        tmem_st16(trow + 128 + 16 * c, dw);
      } else {
        const int j0 = 32 * c;  // first key of the chunk within the tile
        if (cols >= j0 + 32) {
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const float p0 = ex2_approx(fmaf(__uint_as_float(sv[e]), c2, -lse2));
            const float p1 = ex2_approx(fmaf(__uint_as_float(sv[e + 1]), c2, -lse2));
            dw[e / 2] = cvt_bf16x2(p0 * fmaf(vd, __uint_as_float(dv[e]), -d_r),
                                   p1 * fmaf(vd, __uint_as_float(dv[e + 1]), -d_r));
          }
        } else {  // keys past the sequence's end contribute nothing
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            float p0 = ex2_approx(fmaf(__uint_as_float(sv[e]), c2, -lse2));
            float p1 = ex2_approx(fmaf(__uint_as_float(sv[e + 1]), c2, -lse2));
            if (j0 + e >= cols) p0 = 0.0f;
            if (j0 + e + 1 >= cols) p1 = 0.0f;
            dw[e / 2] = cvt_bf16x2(p0 * fmaf(vd, __uint_as_float(dv[e]), -d_r),
                                   p1 * fmaf(vd, __uint_as_float(dv[e + 1]), -d_r));
          }
        }
        tmem_st16(trow + 384 + 16 * c, dw);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(sm.bar(kBbChunk + c));
    }
  }
  // The last commit follows every MMA of the CTA.
  if (n > 0 && !mbar_wait_warp(sm.bar(kBbRFree), (n - 1) & 1, abort_flag)) return false;
  tc_fence_after();
  return true;
}

// dK and dV of one 128-key tile of one (sequence, head).
__global__ void __launch_bounds__(kBwdThreads, 1) attn_bwd_dkdv_kernel(const BwdParams p) {
  extern __shared__ uint8_t bsmem_raw[];
  const BwdSmem sm{reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(bsmem_raw) + 1023) & ~uintptr_t(1023))};
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  const int w = blockIdx.x;
  const int h = w / p.total_k_tiles, g = w - h * p.total_k_tiles;
  const int seq = find_prefix(p.so_k, p.num_seqs, g);
  const int kt = g - __ldg(p.so_k + seq);
  const int k0 = __ldg(p.cu_k + seq), k_len = __ldg(p.cu_k + seq + 1) - k0;
  const int keys = min(128, k_len - kt * 128);
  const int q0 = __ldg(p.cu_q + seq), q_len = __ldg(p.cu_q + seq + 1) - q0;
  const int nq = (q_len + 127) / 128;
  const int so_q = __ldg(p.so_q + seq);
  const int64_t k_atom = (static_cast<int64_t>(__ldg(p.so_k + seq) + kt) * p.heads + h) * 512;

  const uint32_t tm = bwd_setup(sm, tid, warp);
  const volatile int* abort_flag = sm.abort_flag();

  if (warp >= kBwdLoadWarp0) {
    // Loaders: K and V once, then the sequence's query tiles through the two stages.
    const int lw = warp - kBwdLoadWarp0;
    bwd_load_kv_tile(p, k0 + kt * 128, k_atom, h, keys, sm.res0(), sm.res1(), lw, lane);
    fence_proxy_async_smem();
    mbar_arrive(sm.bar(kBbResident));
    bool ok = true;
#pragma unroll 1
    for (int i = 0; i < nq; ++i) {
      const int s = i & 1;
      if (i >= 2 && !mbar_wait_warp(sm.bar(kBbEmpty + s), ((i >> 1) - 1) & 1, abort_flag)) { ok = false; break; }
      bwd_load_q_tile<true>(p, q0 + i * 128, p.q_sf + (static_cast<int64_t>(so_q + i) * p.heads + h) * 512, h,
                            min(128, q_len - i * 128), sm.st0(s), sm.st1(s), sm.dvec(s), sm.lse(s), lw, lane);
      fence_proxy_async_smem();
      mbar_arrive(sm.bar(kBbFull + s));
    }
    if (!ok && lane == 0) bwd_report(sm, 202);
  } else if (warp == kBwdIssueWarp) {
    bool ok = true;
    if (p.debug_stall > 0) {
      // Test hook: wait for a phase of the drain barrier that nothing completes before the drain
      // below, so the wait runs out and the failure path is exercised.
      ok = mbar_wait_warp(sm.bar(kBbDrain), 0, abort_flag);
      if (!ok && lane == 0) bwd_report(sm, 207);
    }
    if (ok && !bwd_issue<true>(sm, tm, nq, lane, abort_flag) && lane == 0) bwd_report(sm, 204);
    bwd_drain(sm, lane);
  } else {
    const int r = tid;  // this thread's key row (TMEM lane)
    const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
    const float c = descale_value(p.q_descale, seq, h) * descale_value(p.k_descale, seq, h) * kBwdRsqrtD;
    const float vd = descale_value(p.v_descale, seq, h);
    const bool ok = bwd_compute<true>(sm, tm, nq, warp, lane, c * kBwdLog2e, vd, 128, abort_flag);
    if (!ok && lane == 0) bwd_report(sm, 200);
    // Epilogue: row r of dV and dK (no query tile: zeros).
    const int64_t out_row = static_cast<int64_t>(k0 + kt * 128 + r) * p.heads + h;
    if (!ok) {
      // (outputs unspecified; the status word reports the failure)
    } else if (nq > 0) {
      bwd_store_rows(tm + lane_addr + 256, vd, r, keys, out_row, p.dv, p.mxfp8_dkv ? p.dv_sf + k_atom : nullptr,
                     p.mxfp8_dkv != 0);
      bwd_store_rows(tm + lane_addr + 384, c, r, keys, out_row, p.dk, p.mxfp8_dkv ? p.dk_sf + k_atom : nullptr,
                     p.mxfp8_dkv != 0);
    } else {
      const size_t bytes = p.mxfp8_dkv ? 128 : 256;
      if (r < keys) {
        memset(static_cast<uint8_t*>(p.dv) + out_row * bytes, 0, bytes);
        memset(static_cast<uint8_t*>(p.dk) + out_row * bytes, 0, bytes);
      }
      if (p.mxfp8_dkv) {  // zero blocks take exponent -127 (byte 0); rows past the keys 0x7F
        const uint32_t word = r < keys ? 0u : 0x7F7F7F7Fu;
        reinterpret_cast<uint32_t*>(p.dv_sf + k_atom)[(r & 31) * 4 + (r >> 5)] = word;
        reinterpret_cast<uint32_t*>(p.dk_sf + k_atom)[(r & 31) * 4 + (r >> 5)] = word;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tm, 512);
  }
}

// dQ of one 128-row query tile of one (sequence, head).
__global__ void __launch_bounds__(kBwdThreads, 1) attn_bwd_dq_kernel(const BwdParams p) {
  extern __shared__ uint8_t bsmem_raw[];
  const BwdSmem sm{reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(bsmem_raw) + 1023) & ~uintptr_t(1023))};
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  const int w = blockIdx.x;
  const int h = w / p.total_q_tiles, g = w - h * p.total_q_tiles;
  const int seq = find_prefix(p.so_q, p.num_seqs, g);
  const int qt = g - __ldg(p.so_q + seq);
  const int q0 = __ldg(p.cu_q + seq), q_len = __ldg(p.cu_q + seq + 1) - q0;
  const int qrows = min(128, q_len - qt * 128);
  const int k0 = __ldg(p.cu_k + seq), k_len = __ldg(p.cu_k + seq + 1) - k0;
  const int nk = (k_len + 127) / 128;
  const int so_k = __ldg(p.so_k + seq);

  const uint32_t tm = bwd_setup(sm, tid, warp);
  const volatile int* abort_flag = sm.abort_flag();

  if (warp >= kBwdLoadWarp0) {
    // Loaders: the query tile (Q, dO, D, LSE) once, then the key tiles through the two stages.
    const int lw = warp - kBwdLoadWarp0;
    bwd_load_q_tile<false>(p, q0 + qt * 128,
                           p.q_sf + (static_cast<int64_t>(__ldg(p.so_q + seq) + qt) * p.heads + h) * 512, h, qrows,
                           sm.res0(), sm.res1(), sm.dvec(0), sm.lse(0), lw, lane);
    fence_proxy_async_smem();
    mbar_arrive(sm.bar(kBbResident));
    bool ok = true;
#pragma unroll 1
    for (int j = 0; j < nk; ++j) {
      const int s = j & 1;
      if (j >= 2 && !mbar_wait_warp(sm.bar(kBbEmpty + s), ((j >> 1) - 1) & 1, abort_flag)) { ok = false; break; }
      bwd_load_kv_tile(p, k0 + j * 128, (static_cast<int64_t>(so_k + j) * p.heads + h) * 512, h,
                       min(128, k_len - j * 128), sm.st0(s), sm.st1(s), lw, lane);
      fence_proxy_async_smem();
      mbar_arrive(sm.bar(kBbFull + s));
    }
    if (!ok && lane == 0) bwd_report(sm, 203);
  } else if (warp == kBwdIssueWarp) {
    if (!bwd_issue<false>(sm, tm, nk, lane, abort_flag) && lane == 0) bwd_report(sm, 205);
    bwd_drain(sm, lane);
  } else {
    const int r = tid;  // this thread's query row (TMEM lane)
    const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
    const float c = descale_value(p.q_descale, seq, h) * descale_value(p.k_descale, seq, h) * kBwdRsqrtD;
    const float vd = descale_value(p.v_descale, seq, h);
    const int last_cols = k_len - (nk - 1) * 128;
    const bool ok = bwd_compute<false>(sm, tm, nk, warp, lane, c * kBwdLog2e, vd, last_cols, abort_flag);
    if (!ok && lane == 0) bwd_report(sm, 201);
    const int64_t tok = q0 + qt * 128 + r;
    if (!ok) {
      // (outputs unspecified; the status word reports the failure)
    } else if (nk > 0) {
      bwd_store_rows(tm + lane_addr + 256, c, r, qrows, tok * p.heads + h, p.dq, nullptr, false);
    } else if (r < qrows) {
      memset(p.dq + (tok * p.heads + h) * 128, 0, 256);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tm, 512);
  }
}
}  // namespace lpfa
