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
// computed in each CTA from dO and O rather than stored. The pipeline is synchronous (load,
// MMA, softmax-style update, MMA), a first version.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "ptx.cuh"

namespace lpfa {

constexpr int kBwdThreads = 128;                 // one thread per tile row
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

// Row r of an MXFP8 tile (128 E4M3 codes at src, the row's 4 scale bytes in sfw) to BF16.
__device__ __forceinline__ void mx_row_to_bf(uint8_t* tile, int r, const uint8_t* src, uint32_t sfw) {
#pragma unroll
  for (int c = 0; c < 8; ++c) {  // 16 codes per step: head_dim [16c, 16c + 16)
    const uint4 raw = *reinterpret_cast<const uint4*>(src + 16 * c);
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
#pragma unroll
    for (int hc = 0; hc < 2; ++hc)
      *reinterpret_cast<uint4*>(tile + bf_tile_offset(r, 2 * c + hc)) =
          make_uint4(outw[4 * hc], outw[4 * hc + 1], outw[4 * hc + 2], outw[4 * hc + 3]);
  }
}

// Row r of a BF16 tile from global BF16 (128 values at src); zeros when src is null.
__device__ __forceinline__ void bf_row_copy(uint8_t* tile, int r, const __nv_bfloat16* src) {
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    const uint4 w = src ? *reinterpret_cast<const uint4*>(src + 8 * c) : make_uint4(0u, 0u, 0u, 0u);
    *reinterpret_cast<uint4*>(tile + bf_tile_offset(r, c)) = w;
  }
}

__device__ __forceinline__ void bf_row_zero(uint8_t* tile, int r) {
#pragma unroll
  for (int c = 0; c < 16; ++c) *reinterpret_cast<uint4*>(tile + bf_tile_offset(r, c)) = make_uint4(0u, 0u, 0u, 0u);
}

// dot(dO_r, O_r) over the 128 BF16 values of a row, in fp32.
__device__ __forceinline__ float bf_row_dot(const __nv_bfloat16* a, const __nv_bfloat16* b) {
  float acc = 0.0f;
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    const uint4 x = *reinterpret_cast<const uint4*>(a + 8 * c);
    const uint4 y = *reinterpret_cast<const uint4*>(b + 8 * c);
    const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc = fmaf(__uint_as_float(xs[i] << 16), __uint_as_float(ys[i] << 16), acc);
      acc = fmaf(__uint_as_float(xs[i] & 0xFFFF0000u), __uint_as_float(ys[i] & 0xFFFF0000u), acc);
    }
  }
  return acc;
}

// BF16 x BF16 -> F32, M = N = 128; a_mn / b_mn: operand is MN-major (else K-major).
__device__ __forceinline__ constexpr uint32_t idesc_bf16(bool a_mn, bool b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (a_mn ? (1u << 15) : 0u) | (b_mn ? (1u << 16) : 0u) |
         (16u << 17) | (8u << 24);
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

// Shared memory of both kernels: four BF16 tiles, two 128-float vectors, one barrier, the TMEM
// slot (plus 1024 bytes of alignment slack).
constexpr uint32_t kBwdSmem = 4 * kBfTile + 2 * 128 * 4 + 16 + 16 + 1024;

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

// dK and dV of one 128-key tile of one (sequence, head).
__global__ void __launch_bounds__(kBwdThreads, 1) attn_bwd_dkdv_kernel(const BwdParams p) {
  extern __shared__ uint8_t bsmem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(bsmem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = smem;
  uint8_t* sV = smem + kBfTile;
  uint8_t* sQ = smem + 2 * kBfTile;
  uint8_t* sDO = smem + 3 * kBfTile;
  float* sLse = reinterpret_cast<float*>(smem + 4 * kBfTile);  // log2 units
  float* sD = sLse + 128;
  uint64_t* bar = reinterpret_cast<uint64_t*>(sD + 128);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bar + 2);
  const int r = threadIdx.x, warp = r >> 5, lane = r & 31;
  const uint32_t leader = lane == 0 ? 1u : 0u;

  const int w = blockIdx.x;
  const int h = w / p.total_k_tiles, g = w - h * p.total_k_tiles;
  const int seq = find_prefix(p.so_k, p.num_seqs, g);
  const int kt = g - __ldg(p.so_k + seq);
  const int k0 = __ldg(p.cu_k + seq), k_len = __ldg(p.cu_k + seq + 1) - k0;
  const int keys = min(128, k_len - kt * 128);
  const int q0 = __ldg(p.cu_q + seq), q_len = __ldg(p.cu_q + seq + 1) - q0;
  const int nq = (q_len + 127) / 128;
  const float c = descale_value(p.q_descale, seq, h) * descale_value(p.k_descale, seq, h) * kBwdRsqrtD;
  const float c2 = c * kBwdLog2e;
  const float vd = descale_value(p.v_descale, seq, h);

  if (r == 0) { mbar_init(bar, 1); mbar_fence_init(); }
  if (warp == 0) tmem_alloc(tslot, 512);
  if (r < keys) {
    const int64_t row = static_cast<int64_t>(k0 + kt * 128 + r) * p.heads + h;
    const int64_t atom = (static_cast<int64_t>(__ldg(p.so_k + seq) + kt) * p.heads + h) * 512;
    const int wi = (r & 31) * 4 + (r >> 5);
    mx_row_to_bf(sK, r, p.k + row * 128, reinterpret_cast<const uint32_t*>(p.k_sf + atom)[wi]);
    mx_row_to_bf(sV, r, p.v + row * 128, reinterpret_cast<const uint32_t*>(p.v_sf + atom)[wi]);
  } else {
    bf_row_zero(sK, r);
    bf_row_zero(sV, r);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = *tslot;
  const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
  const uint32_t sb = smem_u32(smem);
  const uint64_t kK = umma_desc(sb, 16, 1024, kLayoutSw128);
  const uint64_t kV = umma_desc(sb + kBfTile, 16, 1024, kLayoutSw128);
  const uint64_t kQ = umma_desc(sb + 2 * kBfTile, 16, 1024, kLayoutSw128);
  const uint64_t kDO = umma_desc(sb + 3 * kBfTile, 16, 1024, kLayoutSw128);
  const uint64_t mQ = umma_desc(sb + 2 * kBfTile, kBfAtom, 1024, kLayoutSw128);
  const uint64_t mDO = umma_desc(sb + 3 * kBfTile, kBfAtom, 1024, kLayoutSw128);
  constexpr uint32_t idKK = idesc_bf16(false, false), idKM = idesc_bf16(false, true);
  uint32_t phase = 0;
  bool ok = true;
  for (int i = 0; i < nq && ok; ++i) {
    const int qrows = min(128, q_len - i * 128);
    if (r < qrows) {
      const int64_t tok = q0 + i * 128 + r;
      const int64_t row = tok * p.heads + h;
      const int64_t atom = (static_cast<int64_t>(__ldg(p.so_q + seq) + i) * p.heads + h) * 512;
      mx_row_to_bf(sQ, r, p.q + row * 128, reinterpret_cast<const uint32_t*>(p.q_sf + atom)[(r & 31) * 4 + (r >> 5)]);
      bf_row_copy(sDO, r, p.dout + row * 128);
      sD[r] = bf_row_dot(p.dout + row * 128, p.o + row * 128);
      sLse[r] = p.lse[static_cast<int64_t>(h) * p.tq + tok] * kBwdLog2e;
    } else {
      bf_row_zero(sQ, r);
      bf_row_zero(sDO, r);
      sD[r] = 0.0f;
      sLse[r] = INFINITY;  // p = 0 for query rows past the sequence
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) {
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)  // S^T = K Q^T
        mma_f16_ss(tm, bf_kmajor_step(kK, kk), bf_kmajor_step(kQ, kk), idKK, kk > 0 ? 1u : 0u, leader);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)  // dP^T / vd = V dO^T
        mma_f16_ss(tm + 128, bf_kmajor_step(kV, kk), bf_kmajor_step(kDO, kk), idKK, kk > 0 ? 1u : 0u, leader);
      mma_commit(bar, leader);
    }
    // Every thread takes the same decision (a bounded wait that ran out in any thread ends the
    // loop for all, so no thread waits at a block barrier alone).
    if (__syncthreads_or(!mbar_wait(bar, phase, nullptr))) { ok = false; break; }
    phase ^= 1u;
    tc_fence_after();
    // Row r (a key): P^T over S^T's first 64 columns, dS^T over dP^T's, 32 queries at a time
    // (each chunk's BF16 words land on columns already read).
#pragma unroll 1
    for (int cb = 0; cb < 4; ++cb) {
      uint32_t sv[32], dv[32];
      tmem_ld32_sync(tm + lane_addr + cb * 32, sv);
      tmem_ld32_sync(tm + lane_addr + 128 + cb * 32, dv);
      uint32_t pw[16], dw[16];
#pragma unroll
      for (int x = 0; x < 32; x += 2) {
        const int qi = cb * 32 + x;
        float p0 = ex2_approx(__uint_as_float(sv[x]) * c2 - sLse[qi]);
        float p1 = ex2_approx(__uint_as_float(sv[x + 1]) * c2 - sLse[qi + 1]);
        if (r >= keys) { p0 = 0.0f; p1 = 0.0f; }
        const float d0 = p0 * (vd * __uint_as_float(dv[x]) - sD[qi]);
        const float d1 = p1 * (vd * __uint_as_float(dv[x + 1]) - sD[qi + 1]);
        pw[x / 2] = cvt_bf16x2(p0, p1);
        dw[x / 2] = cvt_bf16x2(d0, d1);
      }
      tmem_st16(tm + lane_addr + cb * 16, pw);
      tmem_st16(tm + lane_addr + 128 + cb * 16, dw);
    }
    tmem_wait_st();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) {
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)  // dV / vd += P^T dO
        mma_f16_ts(tm + 256, tm + kk * 8, bf_mnmajor_step(mDO, kk), idKM, (i > 0 || kk > 0) ? 1u : 0u, leader);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)  // dK / c += dS^T Q
        mma_f16_ts(tm + 384, tm + 128 + kk * 8, bf_mnmajor_step(mQ, kk), idKM, (i > 0 || kk > 0) ? 1u : 0u, leader);
      mma_commit(bar, leader);
    }
    if (__syncthreads_or(!mbar_wait(bar, phase, nullptr))) { ok = false; break; }
    phase ^= 1u;
    tc_fence_after();
  }
  if (!ok && r == 0 && atomicCAS(&g_lpfa_status[0], 0, 4 /* LPFA_ERR_TIMEOUT */) == 0)
    atomicExch(&g_lpfa_status[1], 200);
  // Epilogue: row r of dV and dK (no query tile: zeros).
  const int64_t out_row = static_cast<int64_t>(k0 + kt * 128 + r) * p.heads + h;
  const int64_t atom = (static_cast<int64_t>(__ldg(p.so_k + seq) + kt) * p.heads + h) * 512;
  if (!ok) {
    // (outputs unspecified; the status word reports the failure)
  } else if (nq > 0) {
    bwd_store_rows(tm + lane_addr + 256, vd, r, keys, out_row, p.dv, p.mxfp8_dkv ? p.dv_sf + atom : nullptr,
                   p.mxfp8_dkv != 0);
    bwd_store_rows(tm + lane_addr + 384, c, r, keys, out_row, p.dk, p.mxfp8_dkv ? p.dk_sf + atom : nullptr,
                   p.mxfp8_dkv != 0);
  } else if (r < keys) {
    const size_t bytes = p.mxfp8_dkv ? 128 : 256;
    memset(static_cast<uint8_t*>(p.dv) + out_row * bytes, 0, bytes);
    memset(static_cast<uint8_t*>(p.dk) + out_row * bytes, 0, bytes);
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
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(bsmem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sDO = smem + kBfTile;
  uint8_t* sK = smem + 2 * kBfTile;
  uint8_t* sV = smem + 3 * kBfTile;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + 4 * kBfTile + 2 * 128 * 4);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bar + 2);
  const int r = threadIdx.x, warp = r >> 5, lane = r & 31;
  const uint32_t leader = lane == 0 ? 1u : 0u;

  const int w = blockIdx.x;
  const int h = w / p.total_q_tiles, g = w - h * p.total_q_tiles;
  const int seq = find_prefix(p.so_q, p.num_seqs, g);
  const int qt = g - __ldg(p.so_q + seq);
  const int q0 = __ldg(p.cu_q + seq), q_len = __ldg(p.cu_q + seq + 1) - q0;
  const int qrows = min(128, q_len - qt * 128);
  const int k0 = __ldg(p.cu_k + seq), k_len = __ldg(p.cu_k + seq + 1) - k0;
  const int nk = (k_len + 127) / 128;
  const float c = descale_value(p.q_descale, seq, h) * descale_value(p.k_descale, seq, h) * kBwdRsqrtD;
  const float c2 = c * kBwdLog2e;
  const float vd = descale_value(p.v_descale, seq, h);

  if (r == 0) { mbar_init(bar, 1); mbar_fence_init(); }
  if (warp == 0) tmem_alloc(tslot, 512);
  float d_r = 0.0f, lse2 = INFINITY;  // this query row's D and LSE (log2 units); p = 0 past the end
  const int64_t tok = q0 + qt * 128 + r;
  if (r < qrows) {
    const int64_t row = tok * p.heads + h;
    const int64_t atom = (static_cast<int64_t>(__ldg(p.so_q + seq) + qt) * p.heads + h) * 512;
    mx_row_to_bf(sQ, r, p.q + row * 128, reinterpret_cast<const uint32_t*>(p.q_sf + atom)[(r & 31) * 4 + (r >> 5)]);
    bf_row_copy(sDO, r, p.dout + row * 128);
    d_r = bf_row_dot(p.dout + row * 128, p.o + row * 128);
    lse2 = p.lse[static_cast<int64_t>(h) * p.tq + tok] * kBwdLog2e;
  } else {
    bf_row_zero(sQ, r);
    bf_row_zero(sDO, r);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = *tslot;
  const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
  const uint32_t sb = smem_u32(smem);
  const uint64_t kQ = umma_desc(sb, 16, 1024, kLayoutSw128);
  const uint64_t kDO = umma_desc(sb + kBfTile, 16, 1024, kLayoutSw128);
  const uint64_t kK = umma_desc(sb + 2 * kBfTile, 16, 1024, kLayoutSw128);
  const uint64_t kV = umma_desc(sb + 3 * kBfTile, 16, 1024, kLayoutSw128);
  const uint64_t mK = umma_desc(sb + 2 * kBfTile, kBfAtom, 1024, kLayoutSw128);
  constexpr uint32_t idKK = idesc_bf16(false, false), idKM = idesc_bf16(false, true);
  uint32_t phase = 0;
  bool ok = true;
  for (int j = 0; j < nk && ok; ++j) {
    const int keys = min(128, k_len - j * 128);
    if (r < keys) {
      const int64_t row = static_cast<int64_t>(k0 + j * 128 + r) * p.heads + h;
      const int64_t atom = (static_cast<int64_t>(__ldg(p.so_k + seq) + j) * p.heads + h) * 512;
      const int wi = (r & 31) * 4 + (r >> 5);
      mx_row_to_bf(sK, r, p.k + row * 128, reinterpret_cast<const uint32_t*>(p.k_sf + atom)[wi]);
      mx_row_to_bf(sV, r, p.v + row * 128, reinterpret_cast<const uint32_t*>(p.v_sf + atom)[wi]);
    } else {
      bf_row_zero(sK, r);
      bf_row_zero(sV, r);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) {
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)  // S = Q K^T
        mma_f16_ss(tm, bf_kmajor_step(kQ, kk), bf_kmajor_step(kK, kk), idKK, kk > 0 ? 1u : 0u, leader);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)  // dP / vd = dO V^T
        mma_f16_ss(tm + 128, bf_kmajor_step(kDO, kk), bf_kmajor_step(kV, kk), idKK, kk > 0 ? 1u : 0u, leader);
      mma_commit(bar, leader);
    }
    if (__syncthreads_or(!mbar_wait(bar, phase, nullptr))) { ok = false; break; }
    phase ^= 1u;
    tc_fence_after();
    // Row r (a query): dS over S's first 64 columns, 32 keys at a time.
#pragma unroll 1
    for (int cb = 0; cb < 4; ++cb) {
      uint32_t sv[32], dv[32];
      tmem_ld32_sync(tm + lane_addr + cb * 32, sv);
      tmem_ld32_sync(tm + lane_addr + 128 + cb * 32, dv);
      uint32_t dw[16];
#pragma unroll
      for (int x = 0; x < 32; x += 2) {
        const int kj = cb * 32 + x;
        float p0 = ex2_approx(__uint_as_float(sv[x]) * c2 - lse2);
        float p1 = ex2_approx(__uint_as_float(sv[x + 1]) * c2 - lse2);
        if (kj >= keys) p0 = 0.0f;
        if (kj + 1 >= keys) p1 = 0.0f;
        dw[x / 2] = cvt_bf16x2(p0 * (vd * __uint_as_float(dv[x]) - d_r), p1 * (vd * __uint_as_float(dv[x + 1]) - d_r));
      }
      tmem_st16(tm + lane_addr + cb * 16, dw);
    }
    tmem_wait_st();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) {
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)  // dQ / c += dS K
        mma_f16_ts(tm + 256, tm + kk * 8, bf_mnmajor_step(mK, kk), idKM, (j > 0 || kk > 0) ? 1u : 0u, leader);
      mma_commit(bar, leader);
    }
    if (__syncthreads_or(!mbar_wait(bar, phase, nullptr))) { ok = false; break; }
    phase ^= 1u;
    tc_fence_after();
  }
  if (!ok && r == 0 && atomicCAS(&g_lpfa_status[0], 0, 4 /* LPFA_ERR_TIMEOUT */) == 0)
    atomicExch(&g_lpfa_status[1], 201);
  if (!ok) {
    // (outputs unspecified; the status word reports the failure)
  } else if (nk > 0) {
    bwd_store_rows(tm + lane_addr + 256, c, r, qrows, tok * p.heads + h, p.dq, nullptr, false);
  } else if (r < qrows) {
    memset(p.dq + (tok * p.heads + h) * 128, 0, 256);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tm, 512);
  }
}
}  // namespace lpfa
