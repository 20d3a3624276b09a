// dequantize.cuh -- MXFP8 (head_dim orientation) to BF16, exactly.
//
// The inverse of the quantizer's payload/scale pair (LP-FA4 README, "MXFP8 forward and
// backward": E4M3 payload plus one E8M0 power of two per 32-element block along head_dim, in
// 128-token-padded per-sequence storage). Value (t, h, d) = E4M3(payload) * 2^e, e the block's
// scale byte minus 127. E4M3 has 4 significant bits and BF16 8 with FP32's exponent range, so the
// product is a BF16 value whenever it is a normal number (e >= -124 for every E4M3 code); the
// arithmetic is that of the attention kernel's in-kernel V converter (E4M3 -> f16x2 exactly, one
// FP32 multiply by 2^e, one round to nearest even to BF16), so both give the same bits.
//
// The bf16 PV mode uses it to convert V once per (token, head) instead of once per query tile
// that reads it: the attention kernel then reads BF16 V by TMA like BF16 V input.
//
// One CTA per (128-token block, head) tile, 256 threads: thread i owns the 16-element chunk
// i % 8 of rows i / 8 + 32 k (k = 0..3); the 8 threads of a row read its 128 payload bytes and
// write its 256 output bytes as whole lines. The four loads of a thread are issued before any
// conversion, so a CTA keeps 16 KB of reads in flight; 8 CTAs fit on an SM.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "ptx.cuh"
#include "quantize.cuh"

namespace lpfa {

constexpr int kDequantThreads = 256;

struct DequantParams {
  const uint8_t* payload;     // (T, H, 128) E4M3 codes
  const uint8_t* scales;      // (blocks * H) 512-byte atoms
  const int32_t* cu_seqlens;  // device, num_seqs + 1
  const int32_t* scale_off;   // device, num_seqs + 1
  int num_seqs;
  int heads;
  __nv_bfloat16* out;         // (T, H, 128)
};

// 2^e for an E8M0 byte b = e + 127, as an FP32 multiplier; b = 0 (2^-127) is the FP32 subnormal.
__device__ __forceinline__ float e8m0_multiplier(uint32_t b) {
  return b >= 1u ? __uint_as_float(b << 23) : __uint_as_float(0x00400000u);
}

__global__ void __launch_bounds__(kDequantThreads) dequantize_mxfp8_kernel(DequantParams p) {
  const int w = blockIdx.x;
  const int g = w / p.heads;
  const int h = w - g * p.heads;
  const int seq = find_seq(p.scale_off, p.num_seqs, g);
  const int blk = g - __ldg(p.scale_off + seq);
  const int start = __ldg(p.cu_seqlens + seq);
  const int rows_valid = min(128, __ldg(p.cu_seqlens + seq + 1) - start - blk * 128);
  const int64_t tok0 = static_cast<int64_t>(start) + blk * 128;
  const int c = threadIdx.x & 7;    // 16-element chunk of head_dim; scale block c / 2
  const int r0 = threadIdx.x >> 3;  // row within each 32-row quarter
  const uint8_t* atom = p.scales + (static_cast<int64_t>(g) * p.heads + h) * 512;

  uint4 raw[4];
  uint32_t sfb[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int r = r0 + 32 * k;
    if (r < rows_valid) {
      raw[k] = __ldg(reinterpret_cast<const uint4*>(p.payload + ((tok0 + r) * p.heads + h) * 128 + c * 16));
      sfb[k] = __ldg(atom + r0 * 16 + k * 4 + (c >> 1));
    }
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int r = r0 + 32 * k;
    if (r >= rows_valid) continue;
    const float scale = e8m0_multiplier(sfb[k]);
    const uint32_t wv[4] = {raw[k].x, raw[k].y, raw[k].z, raw[k].w};
    uint32_t o[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t h01 = cvt_e4m3x2_to_f16x2(static_cast<uint16_t>(wv[i] & 0xFFFFu));
      const uint32_t h23 = cvt_e4m3x2_to_f16x2(static_cast<uint16_t>(wv[i] >> 16));
      const float2 f01 = __half22float2(*reinterpret_cast<const __half2*>(&h01));
      const float2 f23 = __half22float2(*reinterpret_cast<const __half2*>(&h23));
      o[2 * i] = cvt_bf16x2(f01.x * scale, f01.y * scale);
      o[2 * i + 1] = cvt_bf16x2(f23.x * scale, f23.y * scale);
    }
    uint4* dst = reinterpret_cast<uint4*>(p.out + ((tok0 + r) * p.heads + h) * 128 + c * 16);
    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

}  // namespace lpfa
