// quantize.cuh -- MXFP8 varlen quantizer and the unscaled E4M3 cast of V.
//
// Quantizer (LP-FA4 README, "MXFP8 forward and backward"): per (token, head, 32-element
// block along head_dim) the block maximum picks an E8M0 power of two 2^e (RCEIL: smallest e
// with amax <= 448 * 2^e; FLOOR: floor(log2 amax) - 8; clamp [-127, 127]; amax 0 -> byte 0),
// and the payload is E4M3(x * 2^-e) with one round-to-nearest-even, saturating conversion.
// Scales go to the 128-token-padded per-sequence storage in 512-byte atoms: token row r of a
// 128-token block, block kb, at byte (r % 32) * 16 + (r / 32) * 4 + kb; rows past the end of
// the sequence hold 0x7F.
//
// Cast (FastVideo #1654, "fp8 PV mode for the FA4-FP4 attention path"): E4M3(v) with no scale.
//
// Token orientation (same README: Q, K and V keep both hardware orientations): one E8M0 scale per
// 32 consecutive tokens of one (head, channel), the groups aligned to the sequence start, 4 per
// 128-token block, in the same 512-byte atoms with channel n, group g at (n % 32) * 16 +
// (n / 32) * 4 + g; a partial last group takes its maximum over the tokens it has, a group with
// no token holds 0x7F. The block-scaled MXFP8 PV product reads V this way (K = keys).
//
// One persistent kernel serves both: each CTA walks (128-token block, head) tiles with a stride
// of the grid size. One warp stages each tile (128 token rows of one head) into shared memory
// with a single TMA box load, double buffered, so the next tile is in flight while the
// converting warps work on the current one; they read 16 bytes per lane from shared memory,
// find each 32-element block maximum over 4 lanes with warp shuffles, write 8 payload bytes per
// lane (coalesced 128-byte rows) and one scale byte per block. In the token orientation each
// converting warp owns one 32-token group and a range of channels (consecutive channels on
// consecutive lanes): one pass over the group's rows for the maxima, one to scale, convert and
// store (contiguous payload bytes per row across the warp).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ptx.cuh"

namespace lpfa {

// What quantize_mxfp8_kernel produces.
enum QuantKind : int {
  kQuantHeadDim = 0,  // scales per 32 elements along head_dim
  kQuantCast = 1,     // unscaled E4M3, no scales
  kQuantTokens = 2    // scales per 32 tokens of a channel
};

#ifndef LPFA_QUANT_STAGES_BF16
#define LPFA_QUANT_STAGES_BF16 2
#endif
#ifndef LPFA_QUANT_STAGES_F32
#define LPFA_QUANT_STAGES_F32 2
#endif
// Converting warps per CTA (one more warp stages the tiles): 8 for bf16 input (three CTAs fit
// on an SM), 16 for fp32 input (one CTA per SM, twice the bytes per row).
template <typename T> constexpr int quant_warps() { return sizeof(T) == 2 ? 8 : 16; }
template <typename T> constexpr int quant_threads() { return 32 * quant_warps<T>() + 32; }
// Tiles staged per CTA (input tile: 32 KB for bf16, 64 KB for fp32).
template <typename T> constexpr int quant_stages() {
  return sizeof(T) == 2 ? LPFA_QUANT_STAGES_BF16 : LPFA_QUANT_STAGES_F32;
}

struct QuantParams {
  const void* x;
  int64_t tok_stride;   // elements
  int64_t head_stride;  // elements
  int heads;
  int num_seqs;               // quantizer: varlen metadata
  const int32_t* cu_seqlens;  // device, num_seqs + 1
  const int32_t* scale_off;   // device, num_seqs + 1
  int64_t tokens;             // cast: plain token count (no metadata)
  int num_blocks;             // 128-token blocks (quantizer: total_scale_blocks)
  uint8_t* payload;           // (T, H, 128)
  uint8_t* scales;            // quantizer: (blocks * H) * 512
  int floor_mode;
};

// 8 consecutive elements of a staged row as floats.
template <typename T>
__device__ __forceinline__ void smem_load8(const T* p, float (&v)[8]);

template <>
__device__ __forceinline__ void smem_load8<__nv_bfloat16>(const __nv_bfloat16* p, float (&v)[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

template <>
__device__ __forceinline__ void smem_load8<float>(const float* p, float (&v)[8]) {
  const float4 a = reinterpret_cast<const float4*>(p)[0];
  const float4 b = reinterpret_cast<const float4*>(p)[1];
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

__device__ __forceinline__ int find_seq(const int32_t* prefix, int n, int g) {
  // Largest i with prefix[i] <= g (prefix strictly increasing, prefix[0] = 0).
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(prefix + mid) <= g) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// A tile: 128 token rows of one head (rows >= rows_valid do not exist).
struct QuantTile {
  int64_t tok0;    // first token of the tile
  int rows_valid;
  int h;
  int g;           // 128-token block index (the scale atom's block)
};

template <bool kCast>
__device__ __forceinline__ QuantTile quant_tile(const QuantParams& p, int w) {
  // (kCast: a plain token range without metadata.)
  QuantTile t;
  t.g = w / p.heads;
  t.h = w - t.g * p.heads;
  if (kCast) {
    t.tok0 = static_cast<int64_t>(t.g) * 128;
    const int64_t left = p.tokens - t.tok0;
    t.rows_valid = left < 128 ? static_cast<int>(left) : 128;
  } else {
    const int seq = find_seq(p.scale_off, p.num_seqs, t.g);
    const int blk = t.g - __ldg(p.scale_off + seq);
    const int start = __ldg(p.cu_seqlens + seq);
    const int len = __ldg(p.cu_seqlens + seq + 1) - start;
    t.tok0 = start + blk * 128;
    t.rows_valid = min(128, len - blk * 128);
  }
  return t;
}

// Persistent grid over tiles w = g * heads + h (heads of a token block are adjacent in
// memory). Warps 0..7 convert; warp 8 stages tiles (its own warp, so that computing the next
// tile's bounds and issuing its copies never holds up the converting warps). kKind: see
// QuantKind (the cast writes no scale atoms).
template <typename T, int kKind>
__global__ void __launch_bounds__(quant_threads<T>())
quantize_mxfp8_kernel(const __grid_constant__ CUtensorMap tmap_x, QuantParams p) {
  constexpr bool kCast = kKind == kQuantCast;
  constexpr uint32_t kRowBytes = 128 * sizeof(T);
  constexpr uint32_t kTileBytesIn = 128 * kRowBytes;
  constexpr int kQuantStages = quant_stages<T>();
  constexpr int kQuantWarps = quant_warps<T>();
  constexpr int kQuantThreads = 32 * kQuantWarps;
  constexpr int kRowsPerWarp = 128 / kQuantWarps;
  static_assert(128 % (2 * kQuantWarps) == 0, "rows per converting warp");
  extern __shared__ uint8_t qsmem_raw[];
  uint8_t* qsmem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(qsmem_raw) + 127) & ~uintptr_t(127));
  uint64_t* full = reinterpret_cast<uint64_t*>(qsmem + kQuantStages * kTileBytesIn);
  uint64_t* empty = full + kQuantStages;
  QuantTile* info = reinterpret_cast<QuantTile*>(empty + kQuantStages);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(info + kQuantStages);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int num_tiles = p.num_blocks * p.heads;
  const int G = gridDim.x;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kQuantStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kQuantThreads / 32);
    }
    *abort_flag = 0;
    mbar_fence_init();
  }
  __syncthreads();

  if (warp == kQuantThreads / 32) {
    // ---------------------------------------------------------------- producer
    // One TMA load per tile: the box is 128 rows (tokens) x 128 elements of one head; rows
    // past the end of the tensor read as zero, rows of the next sequence are read but unused.
    if (lane == 0) prefetch_tmap(&tmap_x);
    int n = 0;  // tiles issued
    for (int w = blockIdx.x; w < num_tiles; w += G, ++n) {
      const int b = n % kQuantStages;
      if (!mbar_wait(&empty[b], ((n / kQuantStages) & 1) ^ 1, abort_flag)) break;
      const QuantTile t = quant_tile<kCast>(p, w);
      if (lane == 0) {
        info[b] = t;
        fence_proxy_async_smem();  // the converters' reads of buffer b precede the copy below
        mbar_arrive_expect_tx(&full[b], kTileBytesIn, 1u);
        tma_load_3d(qsmem + b * kTileBytesIn, &tmap_x, &full[b], 0, t.h, static_cast<int32_t>(t.tok0), 1u);
      }
      __syncwarp();
    }
    // Copies still in flight must land before the CTA exits: wait (bounded) for the newest fill
    // of each buffer. In normal operation the converters consumed them already.
    for (int j = (n > kQuantStages ? n - kQuantStages : 0); j < n; ++j)
      mbar_wait(&full[j % kQuantStages], (j / kQuantStages) & 1, nullptr);
    return;
  }

  // ------------------------------------------------------------------ converters
  if (kKind == kQuantTokens) {
    // Warp -> (32-token group g, channel range); lane -> kCh consecutive channels.
    constexpr int kCh = 128 / (32 * (kQuantWarps / 4));  // bf16 (8 warps): 2, fp32 (16): 1
    static_assert(kCh == 1 || kCh == 2, "channels per lane");
    const int g = warp & 3;
    const int c0 = (warp >> 2) * (32 * kCh) + lane * kCh;
    int n = 0;
    for (int w = blockIdx.x; w < num_tiles; w += G, ++n) {
      const int b = n % kQuantStages;
      if (!mbar_wait(&full[b], (n / kQuantStages) & 1, abort_flag)) {
        *abort_flag = 1;
        if (atomicCAS(&g_lpfa_status[0], 0, 4 /* LPFA_ERR_TIMEOUT */) == 0) atomicExch(&g_lpfa_status[1], 100);
        break;
      }
      const QuantTile t = info[b];
      const T* src = reinterpret_cast<const T*>(qsmem + b * kTileBytesIn);
      uint8_t* atom = p.scales + (static_cast<int64_t>(t.g) * p.heads + t.h) * 512;
      const int r0 = 32 * g;
      const int r1 = min(t.rows_valid, r0 + 32);
      float amax[kCh];
#pragma unroll
      for (int c = 0; c < kCh; ++c) amax[c] = 0.f;
#pragma unroll 4
      for (int r = r0; r < r1; ++r) {
        float v[kCh];
        if (kCh == 2) {
          const uint32_t u = *reinterpret_cast<const uint32_t*>(src + r * 128 + c0);
          v[0] = __uint_as_float(u << 16);
          v[kCh - 1] = __uint_as_float(u & 0xFFFF0000u);
        } else {
          v[0] = static_cast<float>(src[r * 128 + c0]);
        }
#pragma unroll
        for (int c = 0; c < kCh; ++c) amax[c] = fmaxf(amax[c], fabsf(v[c]));
      }
      int e[kCh];
      float inv[kCh];
#pragma unroll
      for (int c = 0; c < kCh; ++c) {
        e[c] = e8m0_exponent(amax[c], p.floor_mode);
        inv[c] = __uint_as_float(static_cast<uint32_t>(127 - e[c]) << 23);  // 2^-e, normal
      }
#pragma unroll 4
      for (int r = r0; r < r1; ++r) {
        uint8_t* dst = p.payload + ((t.tok0 + r) * p.heads + t.h) * 128 + c0;
        if (kCh == 2) {
          const uint32_t u = *reinterpret_cast<const uint32_t*>(src + r * 128 + c0);
          *reinterpret_cast<uint16_t*>(dst) =
              cvt_e4m3x2(__uint_as_float(u << 16) * inv[0], __uint_as_float(u & 0xFFFF0000u) * inv[kCh - 1]);
        } else {
          *dst = static_cast<uint8_t>(cvt_e4m3x2(static_cast<float>(src[r * 128 + c0]) * inv[0], 0.0f) & 0xFF);
        }
      }
#pragma unroll
      for (int c = 0; c < kCh; ++c) {
        const int ch = c0 + c;
        atom[(ch & 31) * 16 + (ch >> 5) * 4 + g] = r0 < r1 ? static_cast<uint8_t>(e[c] + 127) : uint8_t{0x7F};
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[b]);
    }
    return;
  }
  const int half = lane >> 4;        // which of the two rows of an iteration
  const int col8 = (lane & 15) * 8;  // first of this lane's 8 elements
  const int kb = (lane & 15) >> 2;   // this lane's 32-element block
  int n = 0;
  for (int w = blockIdx.x; w < num_tiles; w += G, ++n) {
    const int b = n % kQuantStages;
    if (!mbar_wait(&full[b], (n / kQuantStages) & 1, abort_flag)) {
      *abort_flag = 1;
      if (atomicCAS(&g_lpfa_status[0], 0, 4 /* LPFA_ERR_TIMEOUT */) == 0) atomicExch(&g_lpfa_status[1], 100);
      break;
    }
    const QuantTile t = info[b];
    const T* src = reinterpret_cast<const T*>(qsmem + b * kTileBytesIn);
    uint8_t* atom = kCast ? nullptr : p.scales + (static_cast<int64_t>(t.g) * p.heads + t.h) * 512;
#pragma unroll 2
    for (int k = 0; k < kRowsPerWarp / 2; ++k) {
      const int r = warp * kRowsPerWarp + k * 2 + half;
      float v[8];
      if (r < t.rows_valid) {
        smem_load8<T>(src + r * 128 + col8, v);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = 0.f;
      }
      float inv = 1.0f;
      int e = 0;
      if (!kCast) {
        float amax = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
        amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 2));
        e = e8m0_exponent(amax, p.floor_mode);
        inv = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);  // 2^-e, normal
      }
      const uint32_t w0 = cvt_e4m3x2(v[0] * inv, v[1] * inv) |
                          (static_cast<uint32_t>(cvt_e4m3x2(v[2] * inv, v[3] * inv)) << 16);
      const uint32_t w1 = cvt_e4m3x2(v[4] * inv, v[5] * inv) |
                          (static_cast<uint32_t>(cvt_e4m3x2(v[6] * inv, v[7] * inv)) << 16);
      if (r < t.rows_valid)
        *reinterpret_cast<uint2*>(p.payload + ((t.tok0 + r) * p.heads + t.h) * 128 + col8) = make_uint2(w0, w1);
      // One lane per 32-element block writes its scale byte; rows past the sequence end
      // hold 0x7F (scale 1.0).
      if (!kCast && (lane & 3) == 0)
        atom[(r & 31) * 16 + (r >> 5) * 4 + kb] = r < t.rows_valid ? static_cast<uint8_t>(e + 127) : uint8_t{0x7F};
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[b]);
  }
}

template <typename T> constexpr uint32_t quant_smem_bytes() {
  return quant_stages<T>() * (128 * 128 * sizeof(T) + 16 + sizeof(QuantTile)) + 16 + 128;  // + alignment
}

}  // namespace lpfa
