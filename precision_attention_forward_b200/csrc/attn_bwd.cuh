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
// Two kernels, no scratch memory:
//   attn_bwd_dkdv_kernel  one CTA per 128-key tile of a (sequence, head): over the sequence's
//                         query tiles it recomputes S^T = K Q^T and dP^T = V dO^T, forms P^T and
//                         dS^T (one thread per key row) and accumulates dV += P^T dO and
//                         dK += dS^T Q in tensor memory (S^T, dP^T, dV, dK: all 512 columns).
//   attn_bwd_dq_kernel    one CTA per 128-row query tile: over the key tiles it recomputes S and
//                         dP, forms dS (one thread per query row) and accumulates dQ += dS K.
// Each CTA dequantizes its MXFP8 tiles to BF16 in shared memory (exact: E4M3 * 2^e is a BF16
// value) and runs BF16 tcgen05 MMAs, so no scale factors are needed in tensor memory. D is
// computed in each CTA from dO and O rather than stored.
//
// Warp roles (256 threads): warps 0-3 compute (one tile row per thread: the MMA issue from warp
// 0, the TMEM reads and writes of the row updates), warps 4-7 load. The loaders fill a
// two-stage ring of the streamed tiles (Q, dO, D, LSE in the dK/dV kernel; K, V in the dQ
// kernel) with coalesced loads, one 16-byte piece per lane, converting as they store; a stage
// is released by a tcgen05.commit after the last MMA that reads it. The first MMA pair of a
// step runs as two N = 64 halves, so the row updates start after the first half; the second MMA
// pair is issued 32 columns at a time behind the row updates.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "ptx.cuh"

namespace lpfa {

constexpr int kBwdThreads = 256;                 // warps 0-3 compute, warps 4-7 load
constexpr int kBwdCompute = 128;                 // one compute thread per tile row
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
// Rows 64..127 of a K-major tile (the second N = 64 half): 64 rows of 128 bytes into each atom.
constexpr uint64_t kBfHalfRows = (64 * 128) >> 4;

constexpr float kBwdLog2e = 1.4426950408889634f;
constexpr float kBwdRsqrtD = 0.08838834764831845f;  // 1 / sqrt(128)

// Shared memory of both kernels (offsets from the 1024-aligned base):
//   [0, 64K)        the resident pair: K, V (dK/dV kernel) or Q, dO (dQ kernel), BF16 tiles
//   [64K, 192K)     two stages of the streamed pair: Q, dO or K, V
//   [192K, +2K)     per stage: LSE (log2 units) and D, 128 floats each (dK/dV kernel); stage 0
//                   holds the resident query tile's in the dQ kernel
//   then            barriers, the TMEM slot, the abort flag
constexpr uint32_t kBwdOffStage = 2 * kBfTile;
constexpr uint32_t kBwdStageBytes = 2 * kBfTile;
constexpr uint32_t kBwdOffVec = kBwdOffStage + 2 * kBwdStageBytes;
constexpr uint32_t kBwdOffBar = kBwdOffVec + 2 * 2 * 128 * 4;
constexpr uint32_t kBwdNumBars = 8;
constexpr uint32_t kBwdSmem = kBwdOffBar + kBwdNumBars * 8 + 16 + 1024;
static_assert(kBwdSmem <= 227 * 1024, "backward shared memory over the per-CTA limit");

struct BwdSmem {
  uint8_t* base;
  __device__ uint8_t* res0() const { return base; }
  __device__ uint8_t* res1() const { return base + kBfTile; }
  __device__ uint8_t* st0(int s) const { return base + kBwdOffStage + s * kBwdStageBytes; }
  __device__ uint8_t* st1(int s) const { return base + kBwdOffStage + s * kBwdStageBytes + kBfTile; }
  __device__ float* lse(int s) const { return reinterpret_cast<float*>(base + kBwdOffVec + s * 1024); }
  __device__ float* dvec(int s) const { return reinterpret_cast<float*>(base + kBwdOffVec + s * 1024 + 512); }
  // barriers: 0 resident full, 1-2 stage full, 3-4 stage empty, 5-6 first-MMA halves, 7 second MMA
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

// ---------------------------------------------------------------------------------------------
// Loaders (warps 4-7; loader warp lw fills rows [32 lw, 32 lw + 32) of a 128-row tile). Every
// load of a tile is issued before the first store, one 16-byte piece per lane, so a warp has 24
// (query tile) or 16 (key tile) loads in flight; rows >= n are written as zeros.
// ---------------------------------------------------------------------------------------------

// A query tile of head h from token tok0 (n rows): Q dequantized to BF16 with its scale atom sf,
// dO copied, D = dO . O (fp32, lanes of a row reduce by shuffles) and LSE in log2 units (+inf
// past the end, so that p = 0 there).
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
  uint4 dv[16], ov[16];
#pragma unroll
  for (int it = 0; it < 16; ++it) {  // dO and O: 2 rows per step, 16 lanes x 8 values per row
    const int r = rb + 2 * it + (lane >> 4);
    dv[it] = make_uint4(0u, 0u, 0u, 0u);
    ov[it] = dv[it];
    if (r < n) {
      const int64_t off = ((tok0 + r) * p.heads + h) * 128;
      dv[it] = __ldg(reinterpret_cast<const uint4*>(p.dout + off) + (lane & 15));
      ov[it] = __ldg(reinterpret_cast<const uint4*>(p.o + off) + (lane & 15));
    }
  }
  const int rl = rb + lane;
  const float lse2 = rl < n ? __ldg(p.lse + static_cast<int64_t>(h) * p.tq + tok0 + rl) * kBwdLog2e : INFINITY;
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
    float d = bf8_dot(dv[it], ov[it]);
    d += __shfl_xor_sync(0xFFFFFFFFu, d, 8);
    d += __shfl_xor_sync(0xFFFFFFFFu, d, 4);
    d += __shfl_xor_sync(0xFFFFFFFFu, d, 2);
    d += __shfl_xor_sync(0xFFFFFFFFu, d, 1);
    if (c == 0) sD[r] = d;
  }
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

// Barrier setup and TMEM allocation shared by both kernels; returns the TMEM base address.
__device__ __forceinline__ uint32_t bwd_setup(const BwdSmem& sm, int tid, int warp) {
  if (tid == 0) {
    for (int b = 0; b < static_cast<int>(kBwdNumBars); ++b) mbar_init(sm.bar(b), b <= 2 ? 128u : 1u);
    *sm.abort_flag() = 0;
    mbar_fence_init();
  }
  if (warp == 0) tmem_alloc(sm.tslot(), 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  return *sm.tslot();
}

// A wait whose outcome the 128 compute threads share: true when every one of them succeeded
// (named barrier 1), so that all of them take the same branch and none is left at a barrier.
__device__ __forceinline__ bool bwd_group_ok(bool waited) { return !bar_red_or(1, kBwdCompute, !waited); }

__device__ __forceinline__ void bwd_report(const BwdSmem& sm, int site) {
  *reinterpret_cast<volatile int*>(sm.abort_flag()) = 1;
  if (atomicCAS(&g_lpfa_status[0], 0, 4 /* LPFA_ERR_TIMEOUT */) == 0) atomicExch(&g_lpfa_status[1], site);
}

// dK and dV of one 128-key tile of one (sequence, head). TMEM columns: S^T 0-127 (P^T as BF16
// over 0-63), dP^T 128-255 (dS^T over 128-191), dV 256-383, dK 384-511.
// Barriers: 0 K/V loaded, 1-2 query stage loaded, 3-4 stage free, 5-6 S^T/dP^T halves done,
// 7 dV/dK step done.
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
  bool ok = true;

  if (warp >= 4) {
    // Loaders: K and V once, then the sequence's query tiles through the two stages.
    const int lw = warp - 4;
    bwd_load_kv_tile(p, k0 + kt * 128, k_atom, h, keys, sm.res0(), sm.res1(), lw, lane);
    fence_proxy_async_smem();
    mbar_arrive(sm.bar(0));
    for (int i = 0; i < nq; ++i) {
      const int s = i & 1;
      if (i >= 2 && !mbar_wait(sm.bar(3 + s), ((i >> 1) - 1) & 1, abort_flag)) { ok = false; break; }
      bwd_load_q_tile(p, q0 + i * 128, p.q_sf + (static_cast<int64_t>(so_q + i) * p.heads + h) * 512, h,
                      min(128, q_len - i * 128), sm.st0(s), sm.st1(s), sm.dvec(s), sm.lse(s), lw, lane);
      fence_proxy_async_smem();
      mbar_arrive(sm.bar(1 + s));
    }
    if (!ok) bwd_report(sm, 202);
  } else {
    const int r = tid;  // this thread's key row (TMEM lane)
    const uint32_t leader = lane == 0 ? 1u : 0u;
    const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
    const float c = descale_value(p.q_descale, seq, h) * descale_value(p.k_descale, seq, h) * kBwdRsqrtD;
    const float c2 = c * kBwdLog2e;
    const float vd = descale_value(p.v_descale, seq, h);
    const uint32_t sb = smem_u32(sm.base);
    const uint64_t kK = umma_desc(sb, 16, 1024, kLayoutSw128);
    const uint64_t kV = umma_desc(sb + kBfTile, 16, 1024, kLayoutSw128);
    constexpr uint32_t idS = idesc_bf16(false, false, 64), idM = idesc_bf16(false, true);
    ok = bwd_group_ok(mbar_wait(sm.bar(0), 0, abort_flag));
    for (int i = 0; i < nq && ok; ++i) {
      const int s = i & 1;
      const uint32_t stq = sb + kBwdOffStage + s * kBwdStageBytes, stdo = stq + kBfTile;
      bool waited = mbar_wait(sm.bar(1 + s), (i >> 1) & 1, abort_flag);
      // The previous step's dV/dK MMAs read P^T and dS^T from the columns S^T and dP^T overwrite.
      if (i > 0) waited = mbar_wait(sm.bar(7), (i - 1) & 1, abort_flag) && waited;
      if (!bwd_group_ok(waited)) { ok = false; break; }
      tc_fence_after();
      if (warp == 0) {
        const uint64_t kQ = umma_desc(stq, 16, 1024, kLayoutSw128), kDO = umma_desc(stdo, 16, 1024, kLayoutSw128);
#pragma unroll
        for (int half = 0; half < 2; ++half) {  // queries [64 half, 64 half + 64)
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)  // S^T = K Q^T
            mma_f16_ss(tm + 64 * half, bf_kmajor_step(kK, kk), bf_kmajor_step(kQ + half * kBfHalfRows, kk), idS,
                       kk > 0 ? 1u : 0u, leader);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)  // dP^T / vd = V dO^T
            mma_f16_ss(tm + 128 + 64 * half, bf_kmajor_step(kV, kk), bf_kmajor_step(kDO + half * kBfHalfRows, kk),
                       idS, kk > 0 ? 1u : 0u, leader);
          mma_commit(sm.bar(5 + half), leader);
        }
      }
      const float* L = sm.lse(s);
      const float* D = sm.dvec(s);
      const uint64_t mQ = umma_desc(stq, kBfAtom, 1024, kLayoutSw128);
      const uint64_t mDO = umma_desc(stdo, kBfAtom, 1024, kLayoutSw128);
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        if (!bwd_group_ok(mbar_wait(sm.bar(5 + half), i & 1, abort_flag))) { ok = false; break; }
        tc_fence_after();
#pragma unroll 1
        for (int cb = 2 * half; cb < 2 * half + 2; ++cb) {
          // Row r: P^T and dS^T for queries [32 cb, 32 cb + 32); their BF16 words land on
          // columns already read.
          uint32_t sv[32], dv[32];
          tmem_ld32x2_sync(tm + lane_addr + cb * 32, tm + lane_addr + 128 + cb * 32, sv, dv);
          uint32_t pw[16], dw[16];
#pragma unroll
          for (int x = 0; x < 32; x += 4) {
            const float4 l4 = *reinterpret_cast<const float4*>(L + cb * 32 + x);
            const float4 d4 = *reinterpret_cast<const float4*>(D + cb * 32 + x);
            const float p0 = ex2_approx(fmaf(__uint_as_float(sv[x]), c2, -l4.x));
            const float p1 = ex2_approx(fmaf(__uint_as_float(sv[x + 1]), c2, -l4.y));
            const float p2 = ex2_approx(fmaf(__uint_as_float(sv[x + 2]), c2, -l4.z));
            const float p3 = ex2_approx(fmaf(__uint_as_float(sv[x + 3]), c2, -l4.w));
            pw[x / 2] = cvt_bf16x2(p0, p1);
            pw[x / 2 + 1] = cvt_bf16x2(p2, p3);
            dw[x / 2] = cvt_bf16x2(p0 * fmaf(vd, __uint_as_float(dv[x]), -d4.x),
                                   p1 * fmaf(vd, __uint_as_float(dv[x + 1]), -d4.y));
            dw[x / 2 + 1] = cvt_bf16x2(p2 * fmaf(vd, __uint_as_float(dv[x + 2]), -d4.z),
                                       p3 * fmaf(vd, __uint_as_float(dv[x + 3]), -d4.w));
          }
          tmem_st16(tm + lane_addr + cb * 16, pw);
          tmem_st16(tm + lane_addr + 128 + cb * 16, dw);
          tmem_wait_st();
          tc_fence_before();
          named_barrier_sync(2, kBwdCompute);
          if (warp == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 2 * cb; kk < 2 * cb + 2; ++kk) {
              const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
              mma_f16_ts(tm + 256, tm + kk * 8, bf_mnmajor_step(mDO, kk), idM, acc, leader);        // dV/vd += P^T dO
              mma_f16_ts(tm + 384, tm + 128 + kk * 8, bf_mnmajor_step(mQ, kk), idM, acc, leader);  // dK/c += dS^T Q
            }
            if (cb == 3) {
              mma_commit(sm.bar(3 + s), leader);
              mma_commit(sm.bar(7), leader);
            }
          }
        }
      }
    }
    if (ok && nq > 0) {
      ok = bwd_group_ok(mbar_wait(sm.bar(7), (nq - 1) & 1, abort_flag));
      tc_fence_after();
    }
    if (!ok && r == 0) bwd_report(sm, 200);
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

// dQ of one 128-row query tile of one (sequence, head). TMEM columns: S 0-127, dP 128-255,
// dQ 256-383, dS as BF16 384-447 (apart from S, so that the next step's S and dP MMAs need not
// wait for this step's dQ MMAs). Barriers: 0 Q/dO/D/LSE loaded, 1-2 key stage loaded, 3-4 stage
// free, 5-6 S/dP halves done, 7 dQ step done.
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
  bool ok = true;

  if (warp >= 4) {
    // Loaders: the query tile (Q, dO, D, LSE) once, then the key tiles through the two stages.
    const int lw = warp - 4;
    bwd_load_q_tile(p, q0 + qt * 128, p.q_sf + (static_cast<int64_t>(__ldg(p.so_q + seq) + qt) * p.heads + h) * 512,
                    h, qrows, sm.res0(), sm.res1(), sm.dvec(0), sm.lse(0), lw, lane);
    fence_proxy_async_smem();
    mbar_arrive(sm.bar(0));
    for (int j = 0; j < nk; ++j) {
      const int s = j & 1;
      if (j >= 2 && !mbar_wait(sm.bar(3 + s), ((j >> 1) - 1) & 1, abort_flag)) { ok = false; break; }
      bwd_load_kv_tile(p, k0 + j * 128, (static_cast<int64_t>(so_k + j) * p.heads + h) * 512, h,
                       min(128, k_len - j * 128), sm.st0(s), sm.st1(s), lw, lane);
      fence_proxy_async_smem();
      mbar_arrive(sm.bar(1 + s));
    }
    if (!ok) bwd_report(sm, 203);
  } else {
    const int r = tid;  // this thread's query row (TMEM lane)
    const uint32_t leader = lane == 0 ? 1u : 0u;
    const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
    const float c = descale_value(p.q_descale, seq, h) * descale_value(p.k_descale, seq, h) * kBwdRsqrtD;
    const float c2 = c * kBwdLog2e;
    const float vd = descale_value(p.v_descale, seq, h);
    const uint32_t sb = smem_u32(sm.base);
    const uint64_t kQ = umma_desc(sb, 16, 1024, kLayoutSw128);
    const uint64_t kDO = umma_desc(sb + kBfTile, 16, 1024, kLayoutSw128);
    constexpr uint32_t idS = idesc_bf16(false, false, 64), idM = idesc_bf16(false, true);
    ok = bwd_group_ok(mbar_wait(sm.bar(0), 0, abort_flag));
    const float d_r = sm.dvec(0)[r];
    const float lse2 = sm.lse(0)[r];  // +inf past the sequence: p = 0
    for (int j = 0; j < nk && ok; ++j) {
      const int s = j & 1;
      const int keys = min(128, k_len - j * 128);
      const uint32_t stk = sb + kBwdOffStage + s * kBwdStageBytes, stv = stk + kBfTile;
      if (!bwd_group_ok(mbar_wait(sm.bar(1 + s), (j >> 1) & 1, abort_flag))) { ok = false; break; }
      tc_fence_after();
      if (warp == 0) {
        const uint64_t kK = umma_desc(stk, 16, 1024, kLayoutSw128), kV = umma_desc(stv, 16, 1024, kLayoutSw128);
#pragma unroll
        for (int half = 0; half < 2; ++half) {  // keys [64 half, 64 half + 64)
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)  // S = Q K^T
            mma_f16_ss(tm + 64 * half, bf_kmajor_step(kQ, kk), bf_kmajor_step(kK + half * kBfHalfRows, kk), idS,
                       kk > 0 ? 1u : 0u, leader);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)  // dP / vd = dO V^T
            mma_f16_ss(tm + 128 + 64 * half, bf_kmajor_step(kDO, kk), bf_kmajor_step(kV + half * kBfHalfRows, kk),
                       idS, kk > 0 ? 1u : 0u, leader);
          mma_commit(sm.bar(5 + half), leader);
        }
      }
      const uint64_t mK = umma_desc(stk, kBfAtom, 1024, kLayoutSw128);
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        bool waited = mbar_wait(sm.bar(5 + half), j & 1, abort_flag);
        // The previous step's dQ MMAs read dS from the columns this step's dS overwrites.
        if (half == 0 && j > 0) waited = mbar_wait(sm.bar(7), (j - 1) & 1, abort_flag) && waited;
        if (!bwd_group_ok(waited)) { ok = false; break; }
        tc_fence_after();
#pragma unroll 1
        for (int cb = 2 * half; cb < 2 * half + 2; ++cb) {
          uint32_t sv[32], dv[32];
          tmem_ld32x2_sync(tm + lane_addr + cb * 32, tm + lane_addr + 128 + cb * 32, sv, dv);
          uint32_t dw[16];
          if (keys >= 128) {
#pragma unroll
            for (int x = 0; x < 32; x += 2) {
              const float p0 = ex2_approx(fmaf(__uint_as_float(sv[x]), c2, -lse2));
              const float p1 = ex2_approx(fmaf(__uint_as_float(sv[x + 1]), c2, -lse2));
              dw[x / 2] = cvt_bf16x2(p0 * fmaf(vd, __uint_as_float(dv[x]), -d_r),
                                     p1 * fmaf(vd, __uint_as_float(dv[x + 1]), -d_r));
            }
          } else {  // the sequence's last key tile: keys past its end contribute nothing
#pragma unroll
            for (int x = 0; x < 32; x += 2) {
              const int kj = cb * 32 + x;
              float p0 = ex2_approx(fmaf(__uint_as_float(sv[x]), c2, -lse2));
              float p1 = ex2_approx(fmaf(__uint_as_float(sv[x + 1]), c2, -lse2));
              if (kj >= keys) p0 = 0.0f;
              if (kj + 1 >= keys) p1 = 0.0f;
              dw[x / 2] = cvt_bf16x2(p0 * fmaf(vd, __uint_as_float(dv[x]), -d_r),
                                     p1 * fmaf(vd, __uint_as_float(dv[x + 1]), -d_r));
            }
          }
          tmem_st16(tm + lane_addr + 384 + cb * 16, dw);
          tmem_wait_st();
          tc_fence_before();
          named_barrier_sync(2, kBwdCompute);
          if (warp == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 2 * cb; kk < 2 * cb + 2; ++kk)  // dQ / c += dS K
              mma_f16_ts(tm + 256, tm + 384 + kk * 8, bf_mnmajor_step(mK, kk), idM, (j > 0 || kk > 0) ? 1u : 0u,
                         leader);
            if (cb == 3) {
              mma_commit(sm.bar(3 + s), leader);
              mma_commit(sm.bar(7), leader);
            }
          }
        }
      }
    }
    if (ok && nk > 0) {
      ok = bwd_group_ok(mbar_wait(sm.bar(7), (nk - 1) & 1, abort_flag));
      tc_fence_after();
    }
    if (!ok && r == 0) bwd_report(sm, 201);
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
