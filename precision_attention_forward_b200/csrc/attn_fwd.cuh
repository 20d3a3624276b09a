// attn_fwd.cuh -- persistent, warp-specialized MXFP8 attention forward for sm_100a.
//
// Computes, per (sequence, head), O = softmax(Q K^T * qd * kd / sqrt(128)) V * vd and the
// natural-log LSE, for noncausal head_dim 128 over packed variable-length sequences
// (LP-FA4 README, "MXFP8 forward and backward"). Q and K are MXFP8 (E4M3 payload, one E8M0
// scale per 32 elements along head_dim). V is either MXFP8 (bf16 PV mode: dequantized to
// BF16 in shared memory, P rounded to BF16) or an unscaled E4M3 cast (fp8 PV mode of
// FastVideo #1654: no V scales, implicit dequant scale 1.0, output still BF16).
// Absent descales are the literal 1.0f on the same code path (vLLM #63232, "Claims").
//
// Work unit: one 128-row query tile of one (sequence, head). The grid is persistent (one CTA
// per SM); CTA b takes units b, b + G, b + 2G, ... in head-major order so that the CTAs
// running at the same time stream the same K/V through L2.
//
// Warp roles (512 threads):
//   warp 0        TMA producer: Q tile + its scale atom, then K/V tiles (+ atoms) in the
//                 order the MMA warp consumes them (K0, K1, V0, K2, V1, ...).
//   warp 1        TMEM allocator and single-thread MMA issuer:
//                   S[b] = Q K_j^T   tcgen05.mma kind::mxf8f6f4.block_scale (scales in TMEM)
//                   O   += P_j V_j   tcgen05.mma kind::f16 (bf16 PV) or kind::f8f6f4 (fp8 PV)
//                                    with P read from TMEM (it overwrites S in place).
//   warps 4..7    softmax group 0: rows 0..127 of the tile, keys 0..63 of every S tile.
//   warps 8..11   softmax group 1: the same rows, keys 64..127. The two groups exchange
//                 row maxima through shared memory once per tile.
//   warps 12..15  bf16 PV mode only: convert the V tile from MXFP8 to BF16 in shared memory.
//
// Online softmax keeps the running maximum m as an integer in log2 units (ceil of the
// scaled row maximum), so every rescale factor 2^(m_old - m_new) is an exact power of two,
// and rescaling of the O accumulator is needed only when the ceiling moves. In fp8 PV mode
// P is stored as E4M3(2^8 * 2^(t - m)); the factor 2^8 cancels in the final division.
//
// TMEM columns (512 allocated): S/P buffer 0 [0,128), S/P buffer 1 [128,256), O [256,384),
// Q scales (2 stages) [384,392), K scales (2 slots) [392,400).
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
constexpr int kTileM = 128;
constexpr int kTileN = 128;
constexpr int kQStages = 2;
constexpr int kKStages = 3;
constexpr int kVStages = 3;
constexpr int kVbfStages = 2;
constexpr uint32_t kTileBytes = 128 * 128;  // one 128 x 128 fp8 tile
constexpr uint32_t kAtomBytes = 512;

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0;
constexpr uint32_t kColO = 256;
constexpr uint32_t kColSFA = 384;
constexpr uint32_t kColSFB = 392;

// log2(e) / sqrt(128) rounded to fp32: logits in log2 units per unit of Q.K.
constexpr float kLog2eRsqrtD = 0.12751743082459868f;
constexpr float kLn2 = 0.69314718055994531f;

// Diagnostic codes stored in g_lpfa_status[1] when a wait gives up.
enum WaitSite : int {
  kSiteProducerQ = 1, kSiteProducerK, kSiteProducerV, kSiteMmaQ, kSiteMmaK, kSiteMmaP,
  kSiteMmaV, kSiteMmaO, kSiteSoftS, kSiteSoftRed, kSiteSoftPV, kSiteSoftL, kSiteConvV,
  kSiteConvE, kSiteDrain, kSiteDebugStall
};

struct AttnParams {
  const uint8_t* q_sf;
  const uint8_t* k_sf;
  const uint8_t* v_sf;      // bf16 PV mode only
  const int32_t* cu_q;      // meta_q.dev
  const int32_t* so_q;      // meta_q.dev + n + 1 (scale / tile prefix)
  const int32_t* cu_k;
  const int32_t* so_k;
  const float* q_descale;   // nullable
  const float* k_descale;
  const float* v_descale;
  __nv_bfloat16* out;       // (Tq, H, 128)
  float* lse;               // (H, Tq)
  int num_seqs;
  int heads;
  int tq;                   // total query tokens
  int total_q_tiles;        // meta_q.total_scale_blocks
  int num_units;            // heads * total_q_tiles
  int debug_stall;          // test hook: >0 makes the MMA warp wait on a phase that never comes
};

// Shared memory layout (offsets from a 1024-byte aligned base).
struct SmemLayout {
  static constexpr uint32_t q = 0;
  static constexpr uint32_t k = q + kQStages * kTileBytes;
  static constexpr uint32_t v = k + kKStages * kTileBytes;
  static constexpr uint32_t vbf = v + kVStages * kTileBytes;         // 2 x 32 KB (bf16 mode)
  static constexpr uint32_t q_sf = vbf + kVbfStages * 2 * kTileBytes;
  static constexpr uint32_t k_sf = q_sf + kQStages * kAtomBytes;
  static constexpr uint32_t v_sf = k_sf + kKStages * kAtomBytes;
  static constexpr uint32_t red = v_sf + kVStages * kAtomBytes;      // float [2 groups][2 slots][128]
  static constexpr uint32_t lsum = red + 2 * 2 * 128 * 4;             // float [2 groups][128]
  static constexpr uint32_t bars = lsum + 2 * 128 * 4;                // uint64 barriers
  static constexpr uint32_t num_bars = 32;
  static constexpr uint32_t misc = bars + num_bars * 8;               // tmem base, abort flag
  static constexpr uint32_t total = misc + 64;
};
constexpr uint32_t kAttnSmemBytes = SmemLayout::total + 1024;  // + alignment slack

// Barrier indices.
enum Bar : int {
  kBarQFull = 0, kBarQEmpty = 2, kBarKFull = 4, kBarKEmpty = 7, kBarVFull = 10, kBarVEmpty = 13,
  kBarVbfFull = 16, kBarVbfEmpty = 18, kBarSFull = 20, kBarPReady = 22, kBarRed = 24,
  kBarPVDone = 26, kBarOEmpty = 27, kBarLReady = 28, kBarDrain = 29
};

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
         (16u << 17) | (1u << 23) | (8u << 24) | (static_cast<uint32_t>(kb) << 29);
}
// E4M3 x E4M3 -> F32, M=128, N=128, A (P) K-major in TMEM, B (V) MN-major.
constexpr uint32_t kIdescPV8 = (1u << 4) | (1u << 16) | (16u << 17) | (8u << 24);
// BF16 x BF16 -> F32, M=128, N=128, A (P) K-major in TMEM, B (V) MN-major.
constexpr uint32_t kIdescPV16 = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | (16u << 17) | (8u << 24);

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

__device__ __forceinline__ UnitInfo unit_info(const AttnParams& p, int w) {
  UnitInfo u;
  u.h = w / p.total_q_tiles;
  const int g = w - u.h * p.total_q_tiles;
  u.seq = find_prefix(p.so_q, p.num_seqs, g);
  u.sbq = __ldg(p.so_q + u.seq);
  u.qtile = g - u.sbq;
  const int cq0 = __ldg(p.cu_q + u.seq);
  u.q_row0 = cq0 + u.qtile * kTileM;
  u.q_len = __ldg(p.cu_q + u.seq + 1) - cq0;
  u.k_row0 = __ldg(p.cu_k + u.seq);
  u.k_len = __ldg(p.cu_k + u.seq + 1) - u.k_row0;
  u.nkv = (u.k_len + kTileN - 1) / kTileN;
  u.sbk = __ldg(p.so_k + u.seq);
  return u;
}

__device__ __forceinline__ void record_failure(volatile int* abort_flag, int site) {
  *abort_flag = 1;
  if (atomicCAS(&g_lpfa_status[0], 0, 4 /* LPFA_ERR_TIMEOUT */) == 0) atomicExch(&g_lpfa_status[1], site);
}

template <bool kFp8PV>
__global__ void __launch_bounds__(kAttnThreads, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                const __grid_constant__ CUtensorMap tmap_v, const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SmemLayout::bars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SmemLayout::misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SmemLayout::misc + 16);
  float* red = reinterpret_cast<float*>(smem + SmemLayout::red);
  float* lsum = reinterpret_cast<float*>(smem + SmemLayout::lsum);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kQStages; ++i) { mbar_init(&bars[kBarQFull + i], 1); mbar_init(&bars[kBarQEmpty + i], 1); }
    for (int i = 0; i < kKStages; ++i) { mbar_init(&bars[kBarKFull + i], 1); mbar_init(&bars[kBarKEmpty + i], 1); }
    for (int i = 0; i < kVStages; ++i) {
      mbar_init(&bars[kBarVFull + i], 1);
      mbar_init(&bars[kBarVEmpty + i], kFp8PV ? 1 : 4);   // MMA commit, or the 4 converter warps
    }
    for (int i = 0; i < kVbfStages; ++i) { mbar_init(&bars[kBarVbfFull + i], 4); mbar_init(&bars[kBarVbfEmpty + i], 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars[kBarSFull + i], 1);
      mbar_init(&bars[kBarPReady + i], 8);
      mbar_init(&bars[kBarRed + i], 8);
    }
    mbar_init(&bars[kBarPVDone], 1);
    mbar_init(&bars[kBarOEmpty], 8);
    mbar_init(&bars[kBarLReady], 8);
    mbar_init(&bars[kBarDrain], 1);
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
  const uint32_t tmem = *tmem_slot;

  const int G = gridDim.x;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t u = 0, qc = 0, kc = 0, vc = 0;  // units, and fills issued per ring
      bool ok = true;
      auto load_v = [&](const UnitInfo& ui, int jj) -> bool {
        const uint32_t s = vc % kVStages, ph = (vc / kVStages) & 1;
        if (!mbar_wait(&bars[kBarVEmpty + s], ph ^ 1, abort_flag)) { record_failure(abort_flag, kSiteProducerV); return false; }
        mbar_arrive_expect_tx(&bars[kBarVFull + s], kTileBytes + (kFp8PV ? 0 : kAtomBytes));
        tma_load_3d(smem + SmemLayout::v + s * kTileBytes, &tmap_v, &bars[kBarVFull + s], 0, ui.h, ui.k_row0 + jj * kTileN);
        if (!kFp8PV)
          bulk_load(smem + SmemLayout::v_sf + s * kAtomBytes,
                    p.v_sf + (static_cast<int64_t>(ui.sbk + jj) * p.heads + ui.h) * kAtomBytes, kAtomBytes,
                    &bars[kBarVFull + s]);
        ++vc;
        return true;
      };
      for (int w = blockIdx.x; w < p.num_units && ok; w += G, ++u) {
        const UnitInfo ui = unit_info(p, w);
        const uint32_t qs = qc % kQStages, qph = (qc / kQStages) & 1;
        if (!mbar_wait(&bars[kBarQEmpty + qs], qph ^ 1, abort_flag)) { record_failure(abort_flag, kSiteProducerQ); ok = false; break; }
        mbar_arrive_expect_tx(&bars[kBarQFull + qs], kTileBytes + kAtomBytes);
        tma_load_3d(smem + SmemLayout::q + qs * kTileBytes, &tmap_q, &bars[kBarQFull + qs], 0, ui.h, ui.q_row0);
        bulk_load(smem + SmemLayout::q_sf + qs * kAtomBytes,
                  p.q_sf + (static_cast<int64_t>(ui.sbq + ui.qtile) * p.heads + ui.h) * kAtomBytes, kAtomBytes,
                  &bars[kBarQFull + qs]);
        ++qc;
        for (int j = 0; j < ui.nkv && ok; ++j) {
          const uint32_t s = kc % kKStages, ph = (kc / kKStages) & 1;
          if (!mbar_wait(&bars[kBarKEmpty + s], ph ^ 1, abort_flag)) { record_failure(abort_flag, kSiteProducerK); ok = false; break; }
          mbar_arrive_expect_tx(&bars[kBarKFull + s], kTileBytes + kAtomBytes);
          tma_load_3d(smem + SmemLayout::k + s * kTileBytes, &tmap_k, &bars[kBarKFull + s], 0, ui.h, ui.k_row0 + j * kTileN);
          bulk_load(smem + SmemLayout::k_sf + s * kAtomBytes,
                    p.k_sf + (static_cast<int64_t>(ui.sbk + j) * p.heads + ui.h) * kAtomBytes, kAtomBytes,
                    &bars[kBarKFull + s]);
          ++kc;
          if (j >= 1) ok = load_v(ui, j - 1);
        }
        if (ok) ok = load_v(ui, ui.nkv - 1);
      }
      // Drain: every copy issued here must land before the CTA exits. The newest fill of each
      // stage is the last one issued into it; older fills of that stage were consumed already.
      for (uint32_t i = (qc > kQStages ? qc - kQStages : 0); i < qc; ++i)
        if (!mbar_wait(&bars[kBarQFull + i % kQStages], (i / kQStages) & 1, nullptr)) record_failure(abort_flag, kSiteDrain);
      for (uint32_t i = (kc > kKStages ? kc - kKStages : 0); i < kc; ++i)
        if (!mbar_wait(&bars[kBarKFull + i % kKStages], (i / kKStages) & 1, nullptr)) record_failure(abort_flag, kSiteDrain);
      for (uint32_t i = (vc > kVStages ? vc - kVStages : 0); i < vc; ++i)
        if (!mbar_wait(&bars[kBarVFull + i % kVStages], (i / kVStages) & 1, nullptr)) record_failure(abort_flag, kSiteDrain);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const float qd = p.q_descale ? __ldg(p.q_descale) : 1.0f;
      const float kd = p.k_descale ? __ldg(p.k_descale) : 1.0f;
      const int negate = (qd * kd) < 0.0f ? 1 : 0;
      const uint32_t sm_q = smem_u32(smem + SmemLayout::q);
      const uint32_t sm_k = smem_u32(smem + SmemLayout::k);
      const uint32_t sm_v = smem_u32(smem + SmemLayout::v);
      const uint32_t sm_vbf = smem_u32(smem + SmemLayout::vbf);
      const uint32_t sm_qsf = smem_u32(smem + SmemLayout::q_sf);
      const uint32_t sm_ksf = smem_u32(smem + SmemLayout::k_sf);
      uint32_t u = 0, kc = 0, vc = 0, sc = 0;
      bool ok = true;
      if (p.debug_stall > 0) {
        // Test hook: wait for a phase of the drain barrier that nothing completes before the
        // drain below, so the wait runs out and the failure path is exercised.
        if (!mbar_wait(&bars[kBarDrain], 0, abort_flag)) { record_failure(abort_flag, kSiteDebugStall); ok = false; }
      }
      // Issue O += P V for S tile `tile_sc` (tile jj of the current unit).
      auto issue_pv = [&](uint32_t tile_sc, int jj) -> bool {
        const uint32_t b = tile_sc & 1;
        if (!mbar_wait(&bars[kBarPReady + b], (tile_sc >> 1) & 1, abort_flag)) { record_failure(abort_flag, kSiteMmaP); return false; }
        if (jj == 0) {
          if (!mbar_wait(&bars[kBarOEmpty], (u & 1) ^ 1, abort_flag)) { record_failure(abort_flag, kSiteMmaO); return false; }
        }
        const uint32_t p_col = tmem + kColS0 + b * 128;
        if (kFp8PV) {
          const uint32_t s = vc % kVStages, ph = (vc / kVStages) & 1;
          if (!mbar_wait(&bars[kBarVFull + s], ph, abort_flag)) { record_failure(abort_flag, kSiteMmaV); return false; }
          tc_fence_after();
          const uint32_t vbase = sm_v + s * kTileBytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t bdesc = umma_desc(vbase + kk * 4096, kTileBytes, 1024, kLayoutSw128);
            mma_f8f6f4_ts(tmem + kColO, p_col + kk * 8, bdesc, kIdescPV8, (jj > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&bars[kBarVEmpty + s]);
        } else {
          const uint32_t s = vc % kVbfStages, ph = (vc / kVbfStages) & 1;
          if (!mbar_wait(&bars[kBarVbfFull + s], ph, abort_flag)) { record_failure(abort_flag, kSiteMmaV); return false; }
          tc_fence_after();
          const uint32_t vbase = sm_vbf + s * 2 * kTileBytes;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t bdesc = umma_desc(vbase + kk * 2048, kTileBytes, 1024, kLayoutSw128);
            mma_f16_ts(tmem + kColO, p_col + kk * 8, bdesc, kIdescPV16, (jj > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&bars[kBarVbfEmpty + s]);
        }
        mma_commit(&bars[kBarPVDone]);
        ++vc;
        return true;
      };
      for (int w = blockIdx.x; w < p.num_units && ok; w += G, ++u) {
        const UnitInfo ui = unit_info(p, w);
        const uint32_t qs = u % kQStages, qph = (u / kQStages) & 1;
        if (!mbar_wait(&bars[kBarQFull + qs], qph, abort_flag)) { record_failure(abort_flag, kSiteMmaQ); ok = false; break; }
        tc_fence_after();
        const uint32_t sfa = tmem + kColSFA + qs * 4;
        tmem_cp_32x128b_x4(sfa, umma_desc(sm_qsf + qs * kAtomBytes, 0, 128, kLayoutNone));
        const uint32_t qbase = sm_q + qs * kTileBytes;
        for (int j = 0; j < ui.nkv; ++j) {
          const uint32_t s = kc % kKStages, ph = (kc / kKStages) & 1;
          if (!mbar_wait(&bars[kBarKFull + s], ph, abort_flag)) { record_failure(abort_flag, kSiteMmaK); ok = false; break; }
          tc_fence_after();
          const uint32_t sfb = tmem + kColSFB + (kc & 1) * 4;
          tmem_cp_32x128b_x4(sfb, umma_desc(sm_ksf + s * kAtomBytes, 0, 128, kLayoutNone));
          const uint32_t kbase = sm_k + s * kTileBytes;
          const uint32_t d_col = tmem + kColS0 + (sc & 1) * 128;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t adesc = umma_desc(qbase + kk * 32, 16, 1024, kLayoutSw128);
            const uint64_t bdesc = umma_desc(kbase + kk * 32, 16, 1024, kLayoutSw128);
            const uint32_t byte_sel = static_cast<uint32_t>(kk) << 30;
            mma_mxf8f6f4_ss(d_col, adesc, bdesc, idesc_qk(kk, negate), sfa | byte_sel, sfb | byte_sel, kk > 0 ? 1u : 0u);
          }
          mma_commit(&bars[kBarSFull + (sc & 1)]);
          mma_commit(&bars[kBarKEmpty + s]);
          if (j == ui.nkv - 1) mma_commit(&bars[kBarQEmpty + qs]);
          ++kc;
          if (j >= 1 && !issue_pv(sc - 1, j - 1)) { ok = false; break; }
          ++sc;
        }
        if (!ok) break;
        if (!issue_pv(sc - 1, ui.nkv - 1)) { ok = false; break; }
      }
      // Drain: wait until every tcgen05 operation issued by this thread has completed.
      mma_commit(&bars[kBarDrain]);
      if (!mbar_wait(&bars[kBarDrain], 0, nullptr)) record_failure(abort_flag, kSiteDrain);
    }
  } else if (warp >= 4 && warp < 12) {
    // ------------------------------------------------------------------ softmax groups
    const int grp = (warp - 4) >> 2;             // 0: keys 0..63, 1: keys 64..127
    const int quarter = warp & 3;                // TMEM lane quarter of this warp
    const int row = quarter * 32 + lane;         // query row within the tile
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const float qd = p.q_descale ? __ldg(p.q_descale) : 1.0f;
    const float kd = p.k_descale ? __ldg(p.k_descale) : 1.0f;
    const float vd = p.v_descale ? __ldg(p.v_descale) : 1.0f;
    const float cscale = fabsf((qd * kd) * kLog2eRsqrtD);  // sign folded into the QK MMA
    const float pbias = kFp8PV ? 8.0f : 0.0f;
    uint32_t u = 0, sc = 0, pvn = 0;
    bool ok = true;
    for (int w = blockIdx.x; w < p.num_units && ok; w += G, ++u) {
      const UnitInfo ui = unit_info(p, w);
      float m = -INFINITY;  // running max, integer valued, log2 units
      float l = 0.f;
      for (int j = 0; j < ui.nkv; ++j) {
        const uint32_t b = sc & 1;
        if (!mbar_wait(&bars[kBarSFull + b], (sc >> 1) & 1, abort_flag)) { record_failure(abort_flag, kSiteSoftS); ok = false; break; }
        tc_fence_after();
        const uint32_t s_addr = tmem + lane_addr + kColS0 + b * 128 + grp * 64;
        uint32_t ra[32], rb[32];
        tmem_ld32(s_addr, ra);
        tmem_ld32(s_addr + 32, rb);
        tmem_ld_wait();
        float s[64];
#pragma unroll
        for (int i = 0; i < 32; ++i) { s[i] = __uint_as_float(ra[i]); s[32 + i] = __uint_as_float(rb[i]); }
        const int key0 = j * kTileN + grp * 64;
        const bool tail = key0 + 64 > ui.k_len;
        if (tail) {
#pragma unroll
          for (int i = 0; i < 64; ++i) if (key0 + i >= ui.k_len) s[i] = -INFINITY;
        }
        float pmax = s[0];
#pragma unroll
        for (int i = 1; i < 64; ++i) pmax = fmaxf(pmax, s[i]);
        // Exchange the partial maxima of the two groups.
        red[(grp * 2 + b) * 128 + row] = pmax;
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[kBarRed + b]);
        if (!mbar_wait(&bars[kBarRed + b], (sc >> 1) & 1, abort_flag)) { record_failure(abort_flag, kSiteSoftRed); ok = false; break; }
        const float tmax = fmaxf(pmax, red[((grp ^ 1) * 2 + b) * 128 + row]);
        const float m_new = fmaxf(m, ceilf(tmax * cscale));
        const float neg_off = pbias - m_new;
        float psum = 0.f;
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          const float e = ex2_approx(fmaf(s[i], cscale, neg_off));
          s[i] = (tail && key0 + i >= ui.k_len) ? 0.f : e;
          psum += s[i];
        }
        const float alpha = ex2_approx(m - m_new);
        l = l * alpha + psum;
        m = m_new;
        // P overwrites the S buffer: group g writes keys [64g, 64g+64).
        if (kFp8PV) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pk[i] = static_cast<uint32_t>(cvt_e4m3x2(s[4 * i], s[4 * i + 1])) |
                    (static_cast<uint32_t>(cvt_e4m3x2(s[4 * i + 2], s[4 * i + 3])) << 16);
          tmem_st16(tmem + lane_addr + kColS0 + b * 128 + grp * 16, pk);
        } else {
          uint32_t pk[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) pk[i] = cvt_bf16x2(s[2 * i], s[2 * i + 1]);
          tmem_st32(tmem + lane_addr + kColS0 + b * 128 + grp * 32, pk);
        }
        // Rescale this group's half of O when the row ceiling moved (never on the first tile).
        if (j > 0 && __any_sync(0xFFFFFFFFu, alpha != 1.0f)) {
          if (!mbar_wait(&bars[kBarPVDone], (pvn - 1) & 1, abort_flag)) { record_failure(abort_flag, kSiteSoftPV); ok = false; break; }
          tc_fence_after();
          const uint32_t o_addr = tmem + lane_addr + kColO + grp * 64;
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            uint32_t ro[32];
            tmem_ld32(o_addr + half * 32, ro);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) ro[i] = __float_as_uint(__uint_as_float(ro[i]) * alpha);
            tmem_st32(o_addr + half * 32, ro);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[kBarPReady + b]);
        ++sc;
        ++pvn;
      }
      if (!ok) break;
      // ---------------------------------------------------------------- epilogue
      if (!mbar_wait(&bars[kBarPVDone], (pvn - 1) & 1, abort_flag)) { record_failure(abort_flag, kSiteSoftPV); ok = false; break; }
      tc_fence_after();
      lsum[grp * 128 + row] = l;
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kBarLReady]);
      if (!mbar_wait(&bars[kBarLReady], u & 1, abort_flag)) { record_failure(abort_flag, kSiteSoftL); ok = false; break; }
      const float ltot = l + lsum[(grp ^ 1) * 128 + row];
      const float oscale = vd / ltot;
      const uint32_t o_addr = tmem + lane_addr + kColO + grp * 64;
      uint32_t ra[32], rb[32];
      tmem_ld32(o_addr, ra);
      tmem_ld32(o_addr + 32, rb);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kBarOEmpty]);
      const bool valid = ui.qtile * kTileM + row < ui.q_len;
      if (valid) {
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
        if (grp == 0) p.lse[static_cast<int64_t>(ui.h) * p.tq + tok] = (m - pbias + lg2_approx(ltot)) * kLn2;
      }
    }
  } else if (!kFp8PV && warp >= 12) {
    // ------------------------------------------------------------------ V converter (bf16 PV)
    const int t = threadIdx.x - 12 * 32;  // key row of the V tile, 0..127
    const uint32_t sw = static_cast<uint32_t>(t & 7);
    uint32_t u = 0, vc = 0;
    bool ok = true;
    for (int w = blockIdx.x; w < p.num_units && ok; w += G, ++u) {
      const UnitInfo ui = unit_info(p, w);
      for (int j = 0; j < ui.nkv; ++j) {
        const uint32_t s = vc % kVStages, ph = (vc / kVStages) & 1;
        const uint32_t sb = vc % kVbfStages, phb = (vc / kVbfStages) & 1;
        if (!mbar_wait(&bars[kBarVFull + s], ph, abort_flag)) { record_failure(abort_flag, kSiteConvV); ok = false; break; }
        if (!mbar_wait(&bars[kBarVbfEmpty + sb], phb ^ 1, abort_flag)) { record_failure(abort_flag, kSiteConvE); ok = false; break; }
        const uint8_t* src = smem + SmemLayout::v + s * kTileBytes + t * 128;
        const uint32_t sfw = reinterpret_cast<const uint32_t*>(smem + SmemLayout::v_sf + s * kAtomBytes)[(t & 31) * 4 + (t >> 5)];
        uint8_t* dst = smem + SmemLayout::vbf + sb * 2 * kTileBytes + t * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {  // 16 fp8 values: head_dim [16c, 16c + 16)
          const uint4 raw = *reinterpret_cast<const uint4*>(src + ((c ^ sw) << 4));
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

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace lpfa
