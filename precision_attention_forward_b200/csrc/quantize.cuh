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
// Both kernels are HBM-bound streaming kernels: 16-byte vector loads, 8-byte vector stores,
// warp-shuffle maxima over the 4 lanes that hold one 32-element block.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ptx.cuh"

namespace lpfa {

constexpr int kQuantThreads = 256;   // 8 warps; one CTA per (128-token block, head)
constexpr int kRowsPerWarp = 16;     // 128 rows / 8 warps

struct QuantParams {
  const void* x;
  int64_t tok_stride;   // elements
  int64_t head_stride;  // elements
  int heads;
  int num_seqs;
  const int32_t* cu_seqlens;  // device, num_seqs + 1
  const int32_t* scale_off;   // device, num_seqs + 1
  uint8_t* payload;           // (T, H, 128)
  uint8_t* scales;            // (blocks * H) * 512
  int floor_mode;
};

// E8M0 exponent of a non-negative float block maximum.
__device__ __forceinline__ int e8m0_exponent(float amax, int floor_mode) {
  const uint32_t bits = __float_as_uint(amax);
  const int biased = static_cast<int>(bits >> 23);
  if (biased == 0) return -127;  // zero or subnormal maximum: below 2^-126, clamps to -127
  const int binade = biased - 127;
  const uint32_t mant = bits & 0x7FFFFFu;
  // 448 = 1.75 * 2^8: a block whose maximum has mantissa <= 0.75 fits at e = binade - 8.
  int e = floor_mode ? binade - 8 : (mant <= 0x600000u ? binade - 8 : binade - 7);
  return max(-127, min(127, e));
}

// Loads 8 consecutive elements as floats.
template <typename T>
__device__ __forceinline__ void load8(const T* p, float (&v)[8]);

template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* p, float (&v)[8]) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

template <>
__device__ __forceinline__ void load8<float>(const float* p, float (&v)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
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

// grid = (total_scale_blocks, heads). Each CTA quantizes the 128 token rows of one scale
// block of one head and writes that block's 512-byte scale atom.
template <typename T>
__global__ void __launch_bounds__(kQuantThreads)
quantize_mxfp8_kernel(QuantParams p) {
  const int g = blockIdx.x;
  const int h = blockIdx.y;
  const int seq = find_seq(p.scale_off, p.num_seqs, g);
  const int blk = g - __ldg(p.scale_off + seq);
  const int seq_start = __ldg(p.cu_seqlens + seq);
  const int seq_len = __ldg(p.cu_seqlens + seq + 1) - seq_start;
  const int rows_valid = min(128, seq_len - blk * 128);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int half = lane >> 4;        // which of the two rows of an iteration
  const int col8 = (lane & 15) * 8;  // first of this lane's 8 elements
  const T* x = static_cast<const T*>(p.x);
  uint32_t* atom = reinterpret_cast<uint32_t*>(p.scales + (static_cast<int64_t>(g) * p.heads + h) * 512);

  constexpr int kIters = kRowsPerWarp / 2;
  float v[kIters][8];
#pragma unroll
  for (int it = 0; it < kIters; ++it) {
    const int r = warp * kRowsPerWarp + it * 2 + half;
    if (r < rows_valid) {
      const int64_t t = seq_start + blk * 128 + r;
      load8<T>(x + t * p.tok_stride + h * p.head_stride + col8, v[it]);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[it][i] = 0.f;
    }
  }

#pragma unroll
  for (int it = 0; it < kIters; ++it) {
    const int r = warp * kRowsPerWarp + it * 2 + half;
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[it][i]));
    amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 2));
    const int e = e8m0_exponent(amax, p.floor_mode);
    const float inv = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);  // 2^-e, normal
    uint32_t w0 = cvt_e4m3x2(v[it][0] * inv, v[it][1] * inv) |
                  (static_cast<uint32_t>(cvt_e4m3x2(v[it][2] * inv, v[it][3] * inv)) << 16);
    uint32_t w1 = cvt_e4m3x2(v[it][4] * inv, v[it][5] * inv) |
                  (static_cast<uint32_t>(cvt_e4m3x2(v[it][6] * inv, v[it][7] * inv)) << 16);
    // Scale bytes of the row's four blocks live in lanes (row base) + 0, 4, 8, 12.
    const uint32_t byte = static_cast<uint32_t>(e + 127);
    const int base = lane & 16;
    const uint32_t b0 = __shfl_sync(0xFFFFFFFFu, byte, base + 0);
    const uint32_t b1 = __shfl_sync(0xFFFFFFFFu, byte, base + 4);
    const uint32_t b2 = __shfl_sync(0xFFFFFFFFu, byte, base + 8);
    const uint32_t b3 = __shfl_sync(0xFFFFFFFFu, byte, base + 12);
    if (r < rows_valid) {
      const int64_t t = seq_start + blk * 128 + r;
      uint2* dst = reinterpret_cast<uint2*>(p.payload + (t * p.heads + h) * 128 + col8);
      *dst = make_uint2(w0, w1);
      if ((lane & 15) == 0) atom[(r & 31) * 4 + (r >> 5)] = b0 | (b1 << 8) | (b2 << 16) | (b3 << 24);
    } else if ((lane & 15) == 0) {
      atom[(r & 31) * 4 + (r >> 5)] = 0x7F7F7F7Fu;  // pad row: scale 1.0
    }
  }
}

struct CastParams {
  const __nv_bfloat16* v;
  int64_t tok_stride;
  int64_t head_stride;
  int64_t rows;  // tokens * heads
  int heads;
  uint8_t* out;
};

// Grid-stride over (token, head) rows; 16 lanes per 128-element row.
__global__ void __launch_bounds__(256) cast_e4m3_kernel(CastParams p) {
  const int64_t lane_global = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t idx = lane_global; idx < p.rows * 16; idx += stride) {
    const int64_t row = idx >> 4;
    const int col8 = static_cast<int>(idx & 15) * 8;
    const int64_t t = row / p.heads;
    const int h = static_cast<int>(row - t * p.heads);
    float v[8];
    load8<__nv_bfloat16>(p.v + t * p.tok_stride + h * p.head_stride + col8, v);
    const uint32_t w0 = cvt_e4m3x2(v[0], v[1]) | (static_cast<uint32_t>(cvt_e4m3x2(v[2], v[3])) << 16);
    const uint32_t w1 = cvt_e4m3x2(v[4], v[5]) | (static_cast<uint32_t>(cvt_e4m3x2(v[6], v[7])) << 16);
    *reinterpret_cast<uint2*>(p.out + row * 128 + col8) = make_uint2(w0, w1);
  }
}

}  // namespace lpfa
