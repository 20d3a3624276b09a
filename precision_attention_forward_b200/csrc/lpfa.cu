// lpfa.cu -- host side of the C ABI declared in include/lpfa.h: argument validation,
// packed varlen metadata, TMA tensor maps and kernel launches. All kernels live in the
// headers included below; this is the library's single translation unit.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "lpfa.h"
#include "attn_fwd.cuh"
#include "attn_fwd_pp.cuh"
#include "attn_bwd.cuh"
#include "quantize.cuh"
#include "dequantize.cuh"

namespace {

thread_local char g_msg[512] = "";

lpfa_status fail(lpfa_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return st;
}

lpfa_status cuda_fail(cudaError_t e, const char* what) {
  return fail(LPFA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool init = false;
  bool sm100 = false;
  int sms = 0;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

// Returns LPFA_OK and fills *info for the current device, or an error status.
lpfa_status current_device(DeviceInfo* info, int* dev_out = nullptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(LPFA_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.init) {
    int major = 0, minor = 0, sms = 0;
    if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess)
      return cuda_fail(e, "cudaDeviceGetAttribute");
    if ((e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess)
      return cuda_fail(e, "cudaDeviceGetAttribute");
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return cuda_fail(e, "cudaDeviceGetAttribute");
    d.sm100 = (major == 10 && minor == 0);
    d.sms = sms;
    d.init = true;
  }
  *info = d;
  if (dev_out) *dev_out = dev;
  return LPFA_OK;
}

lpfa_status require_sm100(DeviceInfo* info) {
  lpfa_status st = current_device(info);
  if (st != LPFA_OK) return st;
  if (!info->sm100) return fail(LPFA_ERR_UNSUPPORTED, "the current device is not sm_100 (B200)");
  return LPFA_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Tensor map over a packed (tokens, heads, 128) uint8 payload; box = box_rows tokens of one
// head, 128-byte rows with the 128-byte swizzle the UMMA descriptors expect.
lpfa_status payload_tmap(CUtensorMap* map, const void* base, int64_t tokens, int heads, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return fail(LPFA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(heads), static_cast<cuuint64_t>(tokens)};
  cuuint64_t strides[2] = {128, static_cast<cuuint64_t>(heads) * 128};
  cuuint32_t box[3] = {128, 1, box_rows};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(LPFA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return LPFA_OK;
}

// Tensor map over a strided (tokens, heads, 128) input of bf16 or fp32 elements; box = 128
// tokens of one head, no swizzle. A dimension of extent 1 gets a dummy stride (it is never
// stepped over).
lpfa_status input_tmap(CUtensorMap* map, const void* base, bool fp32, int64_t tokens, int heads, int64_t tok_stride,
                       int64_t head_stride) {
  auto fn = encode_fn();
  if (!fn) return fail(LPFA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  const int64_t es = fp32 ? 4 : 2;
  const int64_t hs = heads > 1 ? head_stride * es : 128 * es;
  const int64_t ts = tokens > 1 ? tok_stride * es : 128 * es * heads;
  if (hs <= 0 || ts <= 0) return fail(LPFA_ERR_INVALID_ARG, "strides must be positive");
  cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(heads), static_cast<cuuint64_t>(tokens)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(hs), static_cast<cuuint64_t>(ts)};
  cuuint32_t box[3] = {128, 1, 128};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                  const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(LPFA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return LPFA_OK;
}

// Tensor map over a contiguous (tokens, heads, 128) BF16 V; box = 64 elements (128 bytes) of
// one head x 128 tokens with the 128-byte swizzle: the two boxes of a 128-key tile are the two
// MN-major swizzle atoms of the BF16 PV operand.
lpfa_status bf16_v_tmap(CUtensorMap* map, const void* base, int64_t tokens, int heads) {
  auto fn = encode_fn();
  if (!fn) return fail(LPFA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(heads), static_cast<cuuint64_t>(tokens)};
  cuuint64_t strides[2] = {256, static_cast<cuuint64_t>(heads) * 256};
  cuuint32_t box[3] = {64, 1, 128};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(LPFA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return LPFA_OK;
}

lpfa_status check_meta(const lpfa_varlen_meta* m, const char* name) {
  if (!m) return fail(LPFA_ERR_INVALID_ARG, "%s is NULL", name);
  if (!m->dev) return fail(LPFA_ERR_INVALID_ARG, "%s has no device buffer", name);
  if (m->num_seqs < 1 || m->total_tokens < 1 || m->total_scale_blocks < 1)
    return fail(LPFA_ERR_INVALID_ARG, "%s is empty or was not filled", name);
  return LPFA_OK;
}

}  // namespace

extern "C" {

const char* lpfa_last_error_message(void) { return g_msg; }

const char* lpfa_version(void) { return "lpfa 0.1.0 (sm_100a)"; }

size_t lpfa_meta_dev_ints(int32_t num_seqs) {
  return num_seqs < 1 ? 0 : 2 * (static_cast<size_t>(num_seqs) + 1);
}

size_t lpfa_scale_bytes(const lpfa_varlen_meta* meta, int32_t heads) {
  if (!meta || heads < 1 || meta->total_scale_blocks < 0) return 0;
  return static_cast<size_t>(meta->total_scale_blocks) * static_cast<size_t>(heads) * 512u;
}

lpfa_status lpfa_varlen_meta_fill_host(const int32_t* lengths_host, int32_t num_seqs, int32_t* host_ints,
                                       lpfa_varlen_meta* meta) {
  if (!lengths_host || !host_ints || !meta) return fail(LPFA_ERR_INVALID_ARG, "NULL argument");
  if (num_seqs < 1) return fail(LPFA_ERR_INVALID_ARG, "num_seqs must be >= 1 (got %d)", num_seqs);
  int64_t cu = 0, so = 0;
  int32_t mx = 0;
  int32_t* cu_arr = host_ints;
  int32_t* so_arr = host_ints + num_seqs + 1;
  cu_arr[0] = 0;
  so_arr[0] = 0;
  for (int32_t i = 0; i < num_seqs; ++i) {
    const int32_t len = lengths_host[i];
    if (len < 1) return fail(LPFA_ERR_INVALID_ARG, "sequence %d has length %d; lengths must be >= 1", i, len);
    cu += len;
    so += (len + 127) / 128;
    if (cu > INT32_MAX) return fail(LPFA_ERR_INVALID_ARG, "total token count overflows int32");
    cu_arr[i + 1] = static_cast<int32_t>(cu);
    so_arr[i + 1] = static_cast<int32_t>(so);
    if (len > mx) mx = len;
  }
  meta->num_seqs = num_seqs;
  meta->total_tokens = static_cast<int32_t>(cu);
  meta->total_scale_blocks = static_cast<int32_t>(so);
  meta->max_seqlen = mx;
  return LPFA_OK;
}

lpfa_status lpfa_varlen_meta_from_lengths(const int32_t* lengths_host, int32_t num_seqs, lpfa_varlen_meta* meta,
                                          void* stream) {
  if (!meta) return fail(LPFA_ERR_INVALID_ARG, "meta is NULL");
  if (!meta->dev) return fail(LPFA_ERR_INVALID_ARG, "meta->dev must point to a device buffer");
  if (num_seqs < 1) return fail(LPFA_ERR_INVALID_ARG, "num_seqs must be >= 1 (got %d)", num_seqs);
  std::vector<int32_t> host(lpfa_meta_dev_ints(num_seqs));
  lpfa_varlen_meta tmp = *meta;
  lpfa_status st = lpfa_varlen_meta_fill_host(lengths_host, num_seqs, host.data(), &tmp);
  if (st != LPFA_OK) return st;
  // Pageable source: the runtime stages the bytes before returning, so `host` may go away.
  cudaError_t e = cudaMemcpyAsync(meta->dev, host.data(), host.size() * sizeof(int32_t), cudaMemcpyHostToDevice,
                                  static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyAsync(meta)");
  *meta = tmp;
  return LPFA_OK;
}

// Persistent launch of the streaming quantize/cast kernel: as many CTAs as fit on the SMs
// (shared-memory bound), each walking tiles with the grid stride.
static lpfa_status launch_quant(void (*kernel)(const CUtensorMap, lpfa::QuantParams), uint32_t smem, int threads,
                                const CUtensorMap& tmap, const lpfa::QuantParams& p, int sms, cudaStream_t s,
                                const char* what) {
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, smem);
  if (e != cudaSuccess) return cuda_fail(e, "cudaOccupancyMaxActiveBlocksPerMultiprocessor");
  if (per_sm < 1) return fail(LPFA_ERR_UNSUPPORTED, "%s: kernel does not fit on an SM", what);
  const int64_t tiles = static_cast<int64_t>(p.num_blocks) * p.heads;
  const int64_t grid = tiles < static_cast<int64_t>(per_sm) * sms ? tiles : static_cast<int64_t>(per_sm) * sms;
  kernel<<<static_cast<unsigned>(grid), threads, smem, s>>>(tmap, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, what);
  return LPFA_OK;
}

// Both orientations of the varlen quantizer: scales along head_dim or along the tokens.
static lpfa_status quantize_impl(const void* x, lpfa_in_dtype dt, int64_t tok_stride, int64_t head_stride,
                                 int32_t heads, int32_t head_dim, const lpfa_varlen_meta* meta,
                                 lpfa_scaling_mode mode, uint8_t* payload, uint8_t* scales, void* stream,
                                 bool tokens) {
  if (!x || !payload || !scales) return fail(LPFA_ERR_INVALID_ARG, "NULL tensor pointer");
  if (dt != LPFA_IN_BF16 && dt != LPFA_IN_FP32) return fail(LPFA_ERR_INVALID_ARG, "invalid input dtype %d", dt);
  if (mode != LPFA_SCALE_RCEIL && mode != LPFA_SCALE_FLOOR) return fail(LPFA_ERR_INVALID_ARG, "invalid scaling mode %d", mode);
  if (head_dim != 128) return fail(LPFA_ERR_INVALID_ARG, "head_dim must be 128 (got %d)", head_dim);
  if (heads < 1) return fail(LPFA_ERR_INVALID_ARG, "heads must be >= 1");
  lpfa_status st = check_meta(meta, "meta");
  if (st != LPFA_OK) return st;
  const int vec = dt == LPFA_IN_BF16 ? 8 : 4;
  if (!aligned16(x) || !aligned16(payload) || (tok_stride % vec) || (head_stride % vec))
    return fail(LPFA_ERR_INVALID_ARG, "x/payload must be 16-byte aligned with strides multiple of %d elements", vec);
  if (!aligned16(scales)) return fail(LPFA_ERR_INVALID_ARG, "scales must be 16-byte aligned");
  DeviceInfo info;
  if ((st = require_sm100(&info)) != LPFA_OK) return st;
  lpfa::QuantParams p = {};
  p.x = x;
  p.tok_stride = tok_stride;
  p.head_stride = head_stride;
  p.heads = heads;
  p.num_seqs = meta->num_seqs;
  p.cu_seqlens = meta->dev;
  p.scale_off = meta->dev + meta->num_seqs + 1;
  p.num_blocks = meta->total_scale_blocks;
  p.payload = payload;
  p.scales = scales;
  p.floor_mode = mode == LPFA_SCALE_FLOOR ? 1 : 0;
  if (static_cast<int64_t>(p.num_blocks) * heads > INT32_MAX) return fail(LPFA_ERR_INVALID_ARG, "too many tiles");
  CUtensorMap tm;
  if ((st = input_tmap(&tm, x, dt == LPFA_IN_FP32, meta->total_tokens, heads, tok_stride, head_stride)) != LPFA_OK)
    return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dt == LPFA_IN_BF16) {
    auto kernel = tokens ? lpfa::quantize_mxfp8_kernel<__nv_bfloat16, lpfa::kQuantTokens>
                         : lpfa::quantize_mxfp8_kernel<__nv_bfloat16, lpfa::kQuantHeadDim>;
    return launch_quant(kernel, lpfa::quant_smem_bytes<__nv_bfloat16>(), lpfa::quant_threads<__nv_bfloat16>(), tm,
                        p, info.sms, s, "quantize launch");
  }
  auto kernel = tokens ? lpfa::quantize_mxfp8_kernel<float, lpfa::kQuantTokens>
                       : lpfa::quantize_mxfp8_kernel<float, lpfa::kQuantHeadDim>;
  return launch_quant(kernel, lpfa::quant_smem_bytes<float>(), lpfa::quant_threads<float>(), tm, p, info.sms, s,
                      "quantize launch");
}

lpfa_status lpfa_quantize_mxfp8_varlen(const void* x, lpfa_in_dtype dt, int64_t tok_stride, int64_t head_stride,
                                       int32_t heads, int32_t head_dim, const lpfa_varlen_meta* meta,
                                       lpfa_scaling_mode mode, uint8_t* payload, uint8_t* scales, void* stream) {
  return quantize_impl(x, dt, tok_stride, head_stride, heads, head_dim, meta, mode, payload, scales, stream, false);
}

lpfa_status lpfa_quantize_mxfp8_varlen_tokens(const void* x, lpfa_in_dtype dt, int64_t tok_stride,
                                              int64_t head_stride, int32_t heads, int32_t head_dim,
                                              const lpfa_varlen_meta* meta, lpfa_scaling_mode mode,
                                              uint8_t* payload, uint8_t* scales, void* stream) {
  return quantize_impl(x, dt, tok_stride, head_stride, heads, head_dim, meta, mode, payload, scales, stream, true);
}

lpfa_status lpfa_cast_e4m3(const void* v_bf16, int64_t tok_stride, int64_t head_stride, int64_t tokens,
                           int32_t heads, int32_t head_dim, uint8_t* out, void* stream) {
  if (!v_bf16 || !out) return fail(LPFA_ERR_INVALID_ARG, "NULL tensor pointer");
  if (head_dim != 128) return fail(LPFA_ERR_INVALID_ARG, "head_dim must be 128 (got %d)", head_dim);
  if (tokens < 1 || heads < 1) return fail(LPFA_ERR_INVALID_ARG, "tokens and heads must be >= 1");
  if (!aligned16(v_bf16) || !aligned16(out) || (tok_stride % 8) || (head_stride % 8))
    return fail(LPFA_ERR_INVALID_ARG, "v/out must be 16-byte aligned with strides multiple of 8 elements");
  DeviceInfo info;
  lpfa_status st = require_sm100(&info);
  if (st != LPFA_OK) return st;
  lpfa::QuantParams p = {};
  p.x = v_bf16;
  p.tok_stride = tok_stride;
  p.head_stride = head_stride;
  p.heads = heads;
  p.tokens = tokens;
  const int64_t blocks = (tokens + 127) / 128;
  if (blocks * heads > INT32_MAX) return fail(LPFA_ERR_INVALID_ARG, "too many tiles");
  p.num_blocks = static_cast<int>(blocks);
  p.payload = out;
  CUtensorMap tm;
  if ((st = input_tmap(&tm, v_bf16, false, tokens, heads, tok_stride, head_stride)) != LPFA_OK) return st;
  return launch_quant(lpfa::quantize_mxfp8_kernel<__nv_bfloat16, lpfa::kQuantCast>, lpfa::quant_smem_bytes<__nv_bfloat16>(),
                        lpfa::quant_threads<__nv_bfloat16>(), tm, p,
                      info.sms, static_cast<cudaStream_t>(stream), "cast launch");
}

// The attention kernel moves registers between its warpgroups with setmaxnreg; the split
// adds up to exactly the launch allocation of kLaunchRegs per thread, so a build whose
// register count differs is refused here instead of launched (a larger split than the
// allocation would never be granted). Also raises the dynamic shared memory limit.
static lpfa_status check_attn_kernel(const void* fn, uint32_t smem_bytes) {
  cudaFuncAttributes attr;
  cudaError_t e = cudaFuncGetAttributes(&attr, fn);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncGetAttributes");
  if (attr.numRegs != lpfa::kLaunchRegs)
    return fail(LPFA_ERR_UNSUPPORTED, "attention kernel built with %d registers per thread; its warpgroup register "
                "split needs exactly %d", attr.numRegs, lpfa::kLaunchRegs);
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem_bytes));
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
  return LPFA_OK;
}

// MXFP8 (head_dim orientation) -> BF16 over every token of meta: one CTA per (block, head) tile.
static lpfa_status launch_dequant(const uint8_t* payload, const uint8_t* scales, const lpfa_varlen_meta* meta,
                                  int32_t heads, __nv_bfloat16* out, cudaStream_t s) {
  const int64_t tiles = static_cast<int64_t>(meta->total_scale_blocks) * heads;
  if (tiles > INT32_MAX) return fail(LPFA_ERR_INVALID_ARG, "too many (block, head) tiles");
  lpfa::DequantParams p;
  p.payload = payload;
  p.scales = scales;
  p.cu_seqlens = meta->dev;
  p.scale_off = meta->dev + meta->num_seqs + 1;
  p.num_seqs = meta->num_seqs;
  p.heads = heads;
  p.out = out;
  lpfa::dequantize_mxfp8_kernel<<<static_cast<unsigned>(tiles), lpfa::kDequantThreads, 0, s>>>(p);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "dequantize launch");
  return LPFA_OK;
}

extern "C++" {
// Every PV mode runs over pairs of query tiles (attn_fwd_pp.cuh).
template <int kPv, bool kPerUnit>
static lpfa_status launch_attn_pp(int grid, cudaStream_t s, const CUtensorMap& tq, const CUtensorMap& tk,
                                  const CUtensorMap& tv, const lpfa::AttnParams& p) {
  constexpr uint32_t smem = lpfa::pp::smem_bytes<kPv>();
  const void* fn = reinterpret_cast<const void*>(lpfa::pp::attn_fwd_pp_kernel<kPv, kPerUnit>);
  const lpfa_status st = check_attn_kernel(fn, smem);
  if (st != LPFA_OK) return st;
  lpfa::pp::attn_fwd_pp_kernel<kPv, kPerUnit><<<grid, lpfa::kAttnThreads, smem, s>>>(tq, tk, tv, p);
  return LPFA_OK;
}
}  // extern "C++"

// Internal entry shared with the test hook: debug_stall > 0 forces a bounded wait to run out.
static lpfa_status attn_fwd_impl(const uint8_t* q, const uint8_t* q_sf, const uint8_t* k, const uint8_t* k_sf,
                                 const uint8_t* v, const uint8_t* v_sf, const lpfa_varlen_meta* meta_q,
                                 const lpfa_varlen_meta* meta_k, int32_t heads, int32_t head_dim,
                                 lpfa_pv_mode pv_mode, const lpfa_descale* q_descale,
                                 const lpfa_descale* k_descale, const lpfa_descale* v_descale, void* out_bf16,
                                 float* lse, void* stream, int debug_stall, int shared_q = 0,
                                 bool with_ws = false, void* workspace = nullptr, size_t ws_bytes = 0) {
  if (!q || !q_sf || !k || !k_sf || !v || !out_bf16 || !lse) return fail(LPFA_ERR_INVALID_ARG, "NULL tensor pointer");
  if (pv_mode != LPFA_PV_BF16 && pv_mode != LPFA_PV_FP8 && pv_mode != LPFA_PV_BF16_V && pv_mode != LPFA_PV_MXFP8)
    return fail(LPFA_ERR_INVALID_ARG, "invalid pv_mode %d", pv_mode);
  if (pv_mode == LPFA_PV_FP8 && v_sf) return fail(LPFA_ERR_INVALID_ARG, "fp8 PV mode takes no V scale factors (v_sf must be NULL)");
  if (pv_mode == LPFA_PV_BF16_V && v_sf) return fail(LPFA_ERR_INVALID_ARG, "BF16 V input takes no V scale factors (v_sf must be NULL)");
  if (pv_mode == LPFA_PV_BF16 && !v_sf) return fail(LPFA_ERR_INVALID_ARG, "bf16 PV mode needs the V scale factors (v_sf)");
  if (pv_mode == LPFA_PV_MXFP8 && !v_sf)
    return fail(LPFA_ERR_INVALID_ARG, "MXFP8 PV mode needs V's token-orientation scale factors (v_sf)");
  if (head_dim != 128) return fail(LPFA_ERR_INVALID_ARG, "head_dim must be 128 (got %d)", head_dim);
  if (heads < 1) return fail(LPFA_ERR_INVALID_ARG, "heads must be >= 1");
  for (const lpfa_descale* d : {q_descale, k_descale, v_descale})
    if (d && d->ptr && (d->seq_stride < 0 || d->head_stride < 0))
      return fail(LPFA_ERR_INVALID_ARG, "descale strides must be >= 0");
  lpfa_status st;
  if ((st = check_meta(meta_q, "meta_q")) != LPFA_OK) return st;
  if ((st = check_meta(meta_k, "meta_k")) != LPFA_OK) return st;
  if (shared_q) {
    if (meta_q->num_seqs != 1)
      return fail(LPFA_ERR_INVALID_ARG, "a shared query set is one sequence (meta_q has %d)", meta_q->num_seqs);
  } else if (meta_q->num_seqs != meta_k->num_seqs) {
    return fail(LPFA_ERR_INVALID_ARG, "meta_q has %d sequences but meta_k has %d", meta_q->num_seqs, meta_k->num_seqs);
  }
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(q_sf) || !aligned16(k_sf) ||
      (v_sf && !aligned16(v_sf)) || !aligned16(out_bf16) || !aligned16(lse))
    return fail(LPFA_ERR_INVALID_ARG, "all tensors must be 16-byte aligned");
  // Output rows: the query tokens, or (shared query set) one block of them per K/V sequence.
  const int64_t out_rows = shared_q ? static_cast<int64_t>(meta_k->num_seqs) * meta_q->total_tokens
                                    : static_cast<int64_t>(meta_q->total_tokens);
  const int64_t units = shared_q ? static_cast<int64_t>(meta_k->num_seqs) * heads * ((meta_q->total_scale_blocks + 1) / 2)
                                 : static_cast<int64_t>(heads) * meta_q->total_scale_blocks;
  if (units > INT32_MAX || out_rows * heads * 128 > INT64_MAX / 4 || out_rows > INT32_MAX)
    return fail(LPFA_ERR_INVALID_ARG, "too many query tiles or output rows");
  // bf16 PV over a workspace: V is dequantized once into it, then read as BF16 V input.
  const bool dequant_v = with_ws && pv_mode == LPFA_PV_BF16;
  if (dequant_v) {
    const size_t need = static_cast<size_t>(meta_k->total_tokens) * static_cast<size_t>(heads) * 256u;
    if (!workspace) return fail(LPFA_ERR_INVALID_ARG, "bf16 PV mode needs a workspace of %zu bytes", need);
    if (!aligned16(workspace)) return fail(LPFA_ERR_INVALID_ARG, "the workspace must be 16-byte aligned");
    if (ws_bytes < need)
      return fail(LPFA_ERR_INVALID_ARG, "workspace of %zu bytes is too small (bf16 PV mode needs %zu)", ws_bytes,
                  need);
  }
  DeviceInfo info;
  if ((st = require_sm100(&info)) != LPFA_OK) return st;

  CUtensorMap tq, tk, tv;
  if ((st = payload_tmap(&tq, q, meta_q->total_tokens, heads, lpfa::kTileM)) != LPFA_OK) return st;
  if ((st = payload_tmap(&tk, k, meta_k->total_tokens, heads, lpfa::kTileN)) != LPFA_OK) return st;
  if (pv_mode == LPFA_PV_BF16_V || dequant_v) {
    // BF16 V, contiguous (Tk, H, 128): boxes of 64 elements (128 bytes) x 128 keys, 128-byte swizzle.
    if ((st = bf16_v_tmap(&tv, dequant_v ? workspace : v, meta_k->total_tokens, heads)) != LPFA_OK) return st;
  } else if ((st = payload_tmap(&tv, v, meta_k->total_tokens, heads, lpfa::kTileN)) != LPFA_OK) {
    return st;
  }

  lpfa::AttnParams p;
  p.q_sf = q_sf;
  p.k_sf = k_sf;
  p.v_sf = v_sf;
  p.cu_q = meta_q->dev;
  p.so_q = meta_q->dev + meta_q->num_seqs + 1;
  p.cu_k = meta_k->dev;
  p.so_k = meta_k->dev + meta_k->num_seqs + 1;
  // A missing descale reads the library's device constant 1.0f with zero strides.
  void* one_addr = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&one_addr, lpfa::g_lpfa_one);
  const float* one = static_cast<const float*>(one_addr);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(g_lpfa_one)");
  auto descale = [one](const lpfa_descale* d) {
    lpfa::Descale r{one, 0, 0};
    if (d && d->ptr) r = lpfa::Descale{d->ptr, d->seq_stride, d->head_stride};
    return r;
  };
  p.q_descale = descale(q_descale);
  p.k_descale = descale(k_descale);
  p.v_descale = descale(v_descale);
  p.out = static_cast<__nv_bfloat16*>(out_bf16);
  p.lse = lse;
  p.num_seqs = meta_k->num_seqs;
  p.heads = heads;
  p.tq = static_cast<int>(out_rows);
  p.total_q_tiles = meta_q->total_scale_blocks;
  p.num_units = static_cast<int>(units);
  p.debug_stall = debug_stall;
  p.shared_q = shared_q ? 1 : 0;

  const int grid = static_cast<int>(units < info.sms ? units : info.sms);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool per_unit = (p.q_descale.seq_stride | p.q_descale.head_stride | p.k_descale.seq_stride |
                         p.k_descale.head_stride) != 0;
  if (dequant_v) {
    if ((st = launch_dequant(v, v_sf, meta_k, heads, static_cast<__nv_bfloat16*>(workspace), s)) != LPFA_OK)
      return st;
    p.v_sf = nullptr;
  }
  if (pv_mode == LPFA_PV_FP8) {
    st = per_unit ? launch_attn_pp<lpfa::kPvFp8, true>(grid, s, tq, tk, tv, p)
                  : launch_attn_pp<lpfa::kPvFp8, false>(grid, s, tq, tk, tv, p);
  } else if (pv_mode == LPFA_PV_BF16 && !dequant_v) {
    st = per_unit ? launch_attn_pp<lpfa::kPvBf16Mx, true>(grid, s, tq, tk, tv, p)
                  : launch_attn_pp<lpfa::kPvBf16Mx, false>(grid, s, tq, tk, tv, p);
  } else if (pv_mode == LPFA_PV_MXFP8) {
    st = per_unit ? launch_attn_pp<lpfa::kPvMx, true>(grid, s, tq, tk, tv, p)
                  : launch_attn_pp<lpfa::kPvMx, false>(grid, s, tq, tk, tv, p);
  } else {
    st = per_unit ? launch_attn_pp<lpfa::kPvBf16In, true>(grid, s, tq, tk, tv, p)
                  : launch_attn_pp<lpfa::kPvBf16In, false>(grid, s, tq, tk, tv, p);
  }
  if (st != LPFA_OK) return st;
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "attention launch");
  return LPFA_OK;
}

lpfa_status lpfa_attn_fwd_varlen(const uint8_t* q, const uint8_t* q_sf, const uint8_t* k, const uint8_t* k_sf,
                                 const uint8_t* v, const uint8_t* v_sf, const lpfa_varlen_meta* meta_q,
                                 const lpfa_varlen_meta* meta_k, int32_t heads, int32_t head_dim,
                                 lpfa_pv_mode pv_mode, const float* q_descale, const float* k_descale,
                                 const float* v_descale, void* out_bf16, float* lse, void* stream) {
  const lpfa_descale qd{q_descale, 0, 0}, kd{k_descale, 0, 0}, vd{v_descale, 0, 0};
  return attn_fwd_impl(q, q_sf, k, k_sf, v, v_sf, meta_q, meta_k, heads, head_dim, pv_mode, &qd, &kd, &vd,
                       out_bf16, lse, stream, 0);
}

lpfa_status lpfa_attn_fwd_varlen_descaled(const uint8_t* q, const uint8_t* q_sf, const uint8_t* k,
                                          const uint8_t* k_sf, const uint8_t* v, const uint8_t* v_sf,
                                          const lpfa_varlen_meta* meta_q, const lpfa_varlen_meta* meta_k,
                                          int32_t heads, int32_t head_dim, lpfa_pv_mode pv_mode,
                                          const lpfa_descale* q_descale, const lpfa_descale* k_descale,
                                          const lpfa_descale* v_descale, void* out_bf16, float* lse,
                                          void* stream) {
  return attn_fwd_impl(q, q_sf, k, k_sf, v, v_sf, meta_q, meta_k, heads, head_dim, pv_mode, q_descale, k_descale,
                       v_descale, out_bf16, lse, stream, 0);
}

}  // extern "C"

// Internal entry shared with the test hook: debug_stall > 0 forces a bounded wait to run out.
static lpfa_status attn_bwd_impl(const uint8_t* q, const uint8_t* q_sf, const uint8_t* k, const uint8_t* k_sf,
                                 const uint8_t* v, const uint8_t* v_sf, const void* out_bf16, const void* dout_bf16,
                                 const float* lse, const lpfa_varlen_meta* meta_q, const lpfa_varlen_meta* meta_k,
                                 int32_t heads, int32_t head_dim, const lpfa_descale* q_descale,
                                 const lpfa_descale* k_descale, const lpfa_descale* v_descale, void* dq_bf16,
                                 void* dk, void* dv, uint8_t* dk_sf, uint8_t* dv_sf, int32_t output_mxfp8_dkv,
                                 void* stream, int debug_stall) {
  if (!q || !q_sf || !k || !k_sf || !v || !v_sf || !out_bf16 || !dout_bf16 || !lse || !dq_bf16 || !dk || !dv)
    return fail(LPFA_ERR_INVALID_ARG, "NULL tensor pointer");
  if (output_mxfp8_dkv != 0 && output_mxfp8_dkv != 1) return fail(LPFA_ERR_INVALID_ARG, "output_mxfp8_dkv must be 0 or 1");
  if (output_mxfp8_dkv && (!dk_sf || !dv_sf)) return fail(LPFA_ERR_INVALID_ARG, "MXFP8 dK/dV need dk_sf and dv_sf");
  if (head_dim != 128) return fail(LPFA_ERR_INVALID_ARG, "head_dim must be 128 (got %d)", head_dim);
  if (heads < 1) return fail(LPFA_ERR_INVALID_ARG, "heads must be >= 1");
  for (const lpfa_descale* d : {q_descale, k_descale, v_descale})
    if (d && d->ptr && (d->seq_stride < 0 || d->head_stride < 0))
      return fail(LPFA_ERR_INVALID_ARG, "descale strides must be >= 0");
  lpfa_status st;
  if ((st = check_meta(meta_q, "meta_q")) != LPFA_OK) return st;
  if ((st = check_meta(meta_k, "meta_k")) != LPFA_OK) return st;
  if (meta_q->num_seqs != meta_k->num_seqs)
    return fail(LPFA_ERR_INVALID_ARG, "meta_q has %d sequences but meta_k has %d", meta_q->num_seqs, meta_k->num_seqs);
  for (const void* ptr : {static_cast<const void*>(q), static_cast<const void*>(q_sf), static_cast<const void*>(k),
                          static_cast<const void*>(k_sf), static_cast<const void*>(v), static_cast<const void*>(v_sf),
                          out_bf16, dout_bf16, static_cast<const void*>(lse), static_cast<const void*>(dq_bf16),
                          static_cast<const void*>(dk), static_cast<const void*>(dv)})
    if (!aligned16(ptr)) return fail(LPFA_ERR_INVALID_ARG, "all tensors must be 16-byte aligned");
  if (output_mxfp8_dkv && (!aligned16(dk_sf) || !aligned16(dv_sf)))
    return fail(LPFA_ERR_INVALID_ARG, "all tensors must be 16-byte aligned");
  const int64_t ku = static_cast<int64_t>(heads) * meta_k->total_scale_blocks;
  const int64_t qu = static_cast<int64_t>(heads) * meta_q->total_scale_blocks;
  if (ku > INT32_MAX || qu > INT32_MAX) return fail(LPFA_ERR_INVALID_ARG, "too many tiles");
  DeviceInfo info;
  if ((st = require_sm100(&info)) != LPFA_OK) return st;
  void* one_addr = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&one_addr, lpfa::g_lpfa_one);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(g_lpfa_one)");
  const float* one = static_cast<const float*>(one_addr);
  auto descale = [one](const lpfa_descale* d) {
    lpfa::Descale r{one, 0, 0};
    if (d && d->ptr) r = lpfa::Descale{d->ptr, d->seq_stride, d->head_stride};
    return r;
  };
  lpfa::BwdParams p;
  p.q = q; p.q_sf = q_sf; p.k = k; p.k_sf = k_sf; p.v = v; p.v_sf = v_sf;
  p.o = static_cast<const __nv_bfloat16*>(out_bf16);
  p.dout = static_cast<const __nv_bfloat16*>(dout_bf16);
  p.lse = lse;
  p.cu_q = meta_q->dev;
  p.so_q = meta_q->dev + meta_q->num_seqs + 1;
  p.cu_k = meta_k->dev;
  p.so_k = meta_k->dev + meta_k->num_seqs + 1;
  p.q_descale = descale(q_descale);
  p.k_descale = descale(k_descale);
  p.v_descale = descale(v_descale);
  p.dq = static_cast<__nv_bfloat16*>(dq_bf16);
  p.dk = dk;
  p.dv = dv;
  p.dk_sf = dk_sf;
  p.dv_sf = dv_sf;
  p.num_seqs = meta_q->num_seqs;
  p.heads = heads;
  p.tq = meta_q->total_tokens;
  p.total_q_tiles = meta_q->total_scale_blocks;
  p.total_k_tiles = meta_k->total_scale_blocks;
  p.mxfp8_dkv = output_mxfp8_dkv;
  p.debug_stall = debug_stall;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  for (const void* fn : {reinterpret_cast<const void*>(lpfa::attn_bwd_dkdv_kernel),
                         reinterpret_cast<const void*>(lpfa::attn_bwd_dq_kernel)}) {
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(lpfa::kBwdSmem));
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
  }
  if (ku > 0) {
    // D into the dQ buffer first (read by the dK/dV kernel; the dQ kernel then overwrites it).
    const int64_t rows = static_cast<int64_t>(meta_q->total_tokens) * heads;
    const int64_t blocks = std::min<int64_t>((rows + 15) / 16, static_cast<int64_t>(info.sms) * 16);
    if (blocks > 0) lpfa::attn_bwd_d_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(p);
    lpfa::attn_bwd_dkdv_kernel<<<static_cast<unsigned>(ku), lpfa::kBwdThreads, lpfa::kBwdSmem, s>>>(p);
  }
  if (qu > 0) lpfa::attn_bwd_dq_kernel<<<static_cast<unsigned>(qu), lpfa::kBwdThreads, lpfa::kBwdSmem, s>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "backward launch");
  return LPFA_OK;
}

extern "C" {

lpfa_status lpfa_attn_fwd_shared_q(const uint8_t* q, const uint8_t* q_sf, const uint8_t* k, const uint8_t* k_sf,
                                   const uint8_t* v, const uint8_t* v_sf, const lpfa_varlen_meta* meta_q,
                                   const lpfa_varlen_meta* meta_k, int32_t heads, int32_t head_dim,
                                   lpfa_pv_mode pv_mode, const lpfa_descale* q_descale, const lpfa_descale* k_descale,
                                   const lpfa_descale* v_descale, void* out_bf16, float* lse, void* stream) {
  return attn_fwd_impl(q, q_sf, k, k_sf, v, v_sf, meta_q, meta_k, heads, head_dim, pv_mode, q_descale, k_descale,
                       v_descale, out_bf16, lse, stream, 0, 1);
}

size_t lpfa_attn_fwd_workspace_bytes(const lpfa_varlen_meta* meta_k, int32_t heads, lpfa_pv_mode pv_mode) {
  if (!meta_k || heads < 1 || meta_k->total_tokens < 1 || pv_mode != LPFA_PV_BF16) return 0;
  return static_cast<size_t>(meta_k->total_tokens) * static_cast<size_t>(heads) * 256u;
}

lpfa_status lpfa_attn_fwd_varlen_ws(const uint8_t* q, const uint8_t* q_sf, const uint8_t* k, const uint8_t* k_sf,
                                    const uint8_t* v, const uint8_t* v_sf, const lpfa_varlen_meta* meta_q,
                                    const lpfa_varlen_meta* meta_k, int32_t heads, int32_t head_dim,
                                    lpfa_pv_mode pv_mode, const lpfa_descale* q_descale,
                                    const lpfa_descale* k_descale, const lpfa_descale* v_descale, void* out_bf16,
                                    float* lse, void* workspace, size_t workspace_bytes, void* stream) {
  return attn_fwd_impl(q, q_sf, k, k_sf, v, v_sf, meta_q, meta_k, heads, head_dim, pv_mode, q_descale, k_descale,
                       v_descale, out_bf16, lse, stream, 0, 0, true, workspace, workspace_bytes);
}

lpfa_status lpfa_attn_fwd_shared_q_ws(const uint8_t* q, const uint8_t* q_sf, const uint8_t* k,
                                      const uint8_t* k_sf, const uint8_t* v, const uint8_t* v_sf,
                                      const lpfa_varlen_meta* meta_q, const lpfa_varlen_meta* meta_k, int32_t heads,
                                      int32_t head_dim, lpfa_pv_mode pv_mode, const lpfa_descale* q_descale,
                                      const lpfa_descale* k_descale, const lpfa_descale* v_descale, void* out_bf16,
                                      float* lse, void* workspace, size_t workspace_bytes, void* stream) {
  return attn_fwd_impl(q, q_sf, k, k_sf, v, v_sf, meta_q, meta_k, heads, head_dim, pv_mode, q_descale, k_descale,
                       v_descale, out_bf16, lse, stream, 0, 1, true, workspace, workspace_bytes);
}

lpfa_status lpfa_dequantize_mxfp8_varlen(const uint8_t* payload, const uint8_t* scales, const lpfa_varlen_meta* meta,
                                         int32_t heads, int32_t head_dim, void* out_bf16, void* stream) {
  if (!payload || !scales || !out_bf16) return fail(LPFA_ERR_INVALID_ARG, "NULL tensor pointer");
  if (head_dim != 128) return fail(LPFA_ERR_INVALID_ARG, "head_dim must be 128 (got %d)", head_dim);
  if (heads < 1) return fail(LPFA_ERR_INVALID_ARG, "heads must be >= 1");
  lpfa_status st;
  if ((st = check_meta(meta, "meta")) != LPFA_OK) return st;
  if (!aligned16(payload) || !aligned16(out_bf16))
    return fail(LPFA_ERR_INVALID_ARG, "payload and out must be 16-byte aligned");
  DeviceInfo info;
  if ((st = require_sm100(&info)) != LPFA_OK) return st;
  return launch_dequant(payload, scales, meta, heads, static_cast<__nv_bfloat16*>(out_bf16),
                        static_cast<cudaStream_t>(stream));
}

lpfa_status lpfa_attn_bwd_varlen(const uint8_t* q, const uint8_t* q_sf, const uint8_t* k, const uint8_t* k_sf,
                                 const uint8_t* v, const uint8_t* v_sf, const void* out_bf16, const void* dout_bf16,
                                 const float* lse, const lpfa_varlen_meta* meta_q, const lpfa_varlen_meta* meta_k,
                                 int32_t heads, int32_t head_dim, const lpfa_descale* q_descale,
                                 const lpfa_descale* k_descale, const lpfa_descale* v_descale, void* dq_bf16,
                                 void* dk, void* dv, uint8_t* dk_sf, uint8_t* dv_sf, int32_t output_mxfp8_dkv,
                                 void* stream) {
  return attn_bwd_impl(q, q_sf, k, k_sf, v, v_sf, out_bf16, dout_bf16, lse, meta_q, meta_k, heads, head_dim,
                       q_descale, k_descale, v_descale, dq_bf16, dk, dv, dk_sf, dv_sf, output_mxfp8_dkv, stream, 0);
}

lpfa_status lpfa_attn_bwd_varlen_debug(const uint8_t* q, const uint8_t* q_sf, const uint8_t* k, const uint8_t* k_sf,
                                       const uint8_t* v, const uint8_t* v_sf, const void* out_bf16,
                                       const void* dout_bf16, const float* lse, const lpfa_varlen_meta* meta_q,
                                       const lpfa_varlen_meta* meta_k, int32_t heads, int32_t head_dim,
                                       const lpfa_descale* q_descale, const lpfa_descale* k_descale,
                                       const lpfa_descale* v_descale, void* dq_bf16, void* dk, void* dv,
                                       uint8_t* dk_sf, uint8_t* dv_sf, int32_t output_mxfp8_dkv, void* stream,
                                       int32_t debug_flags) {
  if (debug_flags & ~1) return fail(LPFA_ERR_INVALID_ARG, "unknown debug flags 0x%x", debug_flags);
  return attn_bwd_impl(q, q_sf, k, k_sf, v, v_sf, out_bf16, dout_bf16, lse, meta_q, meta_k, heads, head_dim,
                       q_descale, k_descale, v_descale, dq_bf16, dk, dv, dk_sf, dv_sf, output_mxfp8_dkv, stream,
                       debug_flags & 1);
}

lpfa_status lpfa_attn_fwd_varlen_debug(const uint8_t* q, const uint8_t* q_sf, const uint8_t* k, const uint8_t* k_sf,
                                       const uint8_t* v, const uint8_t* v_sf, const lpfa_varlen_meta* meta_q,
                                       const lpfa_varlen_meta* meta_k, int32_t heads, int32_t head_dim,
                                       lpfa_pv_mode pv_mode, const float* q_descale, const float* k_descale,
                                       const float* v_descale, void* out_bf16, float* lse, void* stream,
                                       int32_t debug_flags) {
  if (debug_flags & ~1) return fail(LPFA_ERR_INVALID_ARG, "unknown debug flags 0x%x", debug_flags);
  const lpfa_descale qd{q_descale, 0, 0}, kd{k_descale, 0, 0}, vd{v_descale, 0, 0};
  return attn_fwd_impl(q, q_sf, k, k_sf, v, v_sf, meta_q, meta_k, heads, head_dim, pv_mode, &qd, &kd, &vd,
                       out_bf16, lse, stream, debug_flags & 1);
}

// ------------------------------------------------------------------ forward without allocation
// bf16 PV needs a BF16 copy of V as scratch. Callers that cannot hand the library device memory get
// it from this file-scope array instead; every GPU that loads the library holds it until exit.
static __device__ __align__(256) uint8_t g_noalloc_scratch[LPFA_NOALLOC_SCRATCH_BYTES];

namespace {
void* g_noalloc_ptr[kMaxDevices] = {};
std::mutex g_noalloc_mu;

// The scratch array's device address on the current device. In host code the array's name is only
// a host-side stand-in, so the address is looked up once per device (with it current) and kept.
lpfa_status noalloc_scratch(void** out) {
  DeviceInfo info;
  int dev = 0;
  lpfa_status st = current_device(&info, &dev);
  if (st != LPFA_OK) return st;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(no-allocation scratch)");
    g_noalloc_ptr[dev] = ptr;
  }
  *out = g_noalloc_ptr[dev];
  return LPFA_OK;
}
}  // namespace

lpfa_status lpfa_attn_fwd_varlen_noalloc(const uint8_t* q, const uint8_t* q_sf, const uint8_t* k,
                                         const uint8_t* k_sf, const uint8_t* v, const uint8_t* v_sf,
                                         const lpfa_varlen_meta* meta_q, const lpfa_varlen_meta* meta_k,
                                         int32_t heads, int32_t head_dim, lpfa_pv_mode pv_mode,
                                         const lpfa_descale* q_descale, const lpfa_descale* k_descale,
                                         const lpfa_descale* v_descale, void* out_bf16, float* lse, void* stream) {
  const size_t need = lpfa_attn_fwd_workspace_bytes(meta_k, heads, pv_mode);
  if (need > static_cast<size_t>(LPFA_NOALLOC_SCRATCH_BYTES))
    return fail(LPFA_ERR_INVALID_ARG,
                "lpfa_attn_fwd_varlen_noalloc: bf16 PV over %d key tokens x %d heads needs %zu bytes of scratch; "
                "its fixed scratch holds %zu (key tokens x heads <= %zu)",
                meta_k->total_tokens, heads, need, static_cast<size_t>(LPFA_NOALLOC_SCRATCH_BYTES),
                static_cast<size_t>(LPFA_NOALLOC_SCRATCH_BYTES) / 256u);
  void* scratch = nullptr;
  if (need > 0) {
    const lpfa_status st = noalloc_scratch(&scratch);
    if (st != LPFA_OK) return st;
  }
  return attn_fwd_impl(q, q_sf, k, k_sf, v, v_sf, meta_q, meta_k, heads, head_dim, pv_mode, q_descale, k_descale,
                       v_descale, out_bf16, lse, stream, 0, 0, true, scratch, static_cast<size_t>(LPFA_NOALLOC_SCRATCH_BYTES));
}

lpfa_status lpfa_device_status(void* stream, int32_t* detail) {
  if (detail) *detail = 0;
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int32_t word[2] = {0, 0};
  e = cudaMemcpyFromSymbol(word, lpfa::g_lpfa_status, sizeof(word));
  if (e != cudaSuccess) return cuda_fail(e, "reading the device status word");
  if (word[0] != 0) {
    const int32_t zero[2] = {0, 0};
    e = cudaMemcpyToSymbol(lpfa::g_lpfa_status, zero, sizeof(zero));
    if (e != cudaSuccess) return cuda_fail(e, "resetting the device status word");
    if (detail) *detail = word[1];
    return fail(LPFA_ERR_TIMEOUT, "a kernel gave up waiting on a barrier (site %d)", word[1]);
  }
  return LPFA_OK;
}

}  // extern "C"
