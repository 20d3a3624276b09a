/*
 * lpfa.h -- C ABI of the block-scaled low-precision FlashAttention forward library
 * (MXFP8 quantization of packed variable-length Q/K/V followed by a noncausal
 * head-dim-128 multi-head attention forward with online softmax, BF16 O and fp32 LSE).
 *
 * Conventions shared by every call
 * --------------------------------
 * - All buffers are owned by the caller. The library never allocates device or
 *   pinned memory. Pointers named *_dev, and every tensor argument, are device
 *   pointers; lengths_host is a host pointer.
 * - Work is enqueued asynchronously on `stream` (a cudaStream_t passed as void*;
 *   NULL is the legacy default stream). Outputs are valid once the stream has
 *   reached the call. Host arrays are read before the call returns.
 * - Every call returns an lpfa_status. Nothing is thrown across the ABI. On a
 *   non-OK status nothing has been enqueued, except for LPFA_ERR_CUDA after a
 *   launch; lpfa_last_error_message() describes the last failure of the calling
 *   thread.
 * - Packed layout: a tensor of T tokens and H heads has shape (T, H, 128); the
 *   tokens of sequence i are rows [cu_seqlens[i], cu_seqlens[i+1]).
 * - Only head_dim 128 is supported; any other value returns LPFA_ERR_INVALID_ARG.
 *
 * Sources. "LP-FA4 README" is the README of the LP-FA4 low-precision FlashAttention-4
 * kernels (facebookresearch ads_model_kernel_library, lp_fa4/README.md). "FastVideo
 * #1654" is the FastVideo pull request "fp8 PV mode for the FA4-FP4 attention path".
 * "vLLM #63232" is the vLLM pull request "FA4: no FP8 descale for a unit per-tensor
 * scale".
 */
#ifndef LPFA_H
#define LPFA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__) || defined(__clang__)
#define LPFA_API __attribute__((visibility("default")))
#else
#define LPFA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LPFA_OK = 0,
  LPFA_ERR_INVALID_ARG = 1,   /* bad enum, size, pointer, alignment or metadata */
  LPFA_ERR_UNSUPPORTED = 2,   /* current device is not sm_100 */
  LPFA_ERR_CUDA = 3,          /* a CUDA runtime call or kernel launch failed */
  LPFA_ERR_TIMEOUT = 4        /* a kernel gave up waiting on one of its own barriers */
} lpfa_status;

typedef enum { LPFA_IN_BF16 = 0, LPFA_IN_FP32 = 1 } lpfa_in_dtype;
typedef enum { LPFA_SCALE_RCEIL = 0, LPFA_SCALE_FLOOR = 1 } lpfa_scaling_mode;
typedef enum { LPFA_PV_BF16 = 0, LPFA_PV_FP8 = 1, LPFA_PV_BF16_V = 2, LPFA_PV_MXFP8 = 3 } lpfa_pv_mode;

/*
 * Packed variable-length metadata (LP-FA4 README, "MXFP8 forward and backward":
 * Mxfp8VarlenMeta.from_lengths; each sequence gets independent scale storage padded
 * to a multiple of 128 tokens).
 *
 * `dev` points to a caller-owned device int32 buffer of lpfa_meta_dev_ints(num_seqs)
 * entries holding two arrays of num_seqs + 1 entries each, in this order:
 *   cu_seqlens[i]   first token of sequence i (cu_seqlens[n] = total_tokens);
 *   scale_off[i]    first 128-token scale block of sequence i,
 *                   scale_off[i+1] - scale_off[i] = ceil(len_i / 128). The same prefix
 *                   numbers the 128-row attention tiles of each sequence.
 */
typedef struct {
  int32_t num_seqs;
  int32_t total_tokens;
  int32_t total_scale_blocks;  /* scale_off[num_seqs] */
  int32_t max_seqlen;
  int32_t* dev;
} lpfa_varlen_meta;

/* Number of int32 entries `dev` must hold for num_seqs sequences: 2 * (num_seqs + 1). */
LPFA_API size_t lpfa_meta_dev_ints(int32_t num_seqs);

/*
 * Host-only metadata builder: computes the scalar fields of `meta` and writes the two
 * arrays (layout as for `dev`) into host_ints, which must hold lpfa_meta_dev_ints(num_seqs)
 * entries. meta->dev is left unchanged. Errors: num_seqs < 1, a length < 1, a total that
 * overflows int32, or a NULL pointer -> LPFA_ERR_INVALID_ARG.
 */
LPFA_API lpfa_status lpfa_varlen_meta_fill_host(const int32_t* lengths_host, int32_t num_seqs,
                                       int32_t* host_ints, lpfa_varlen_meta* meta);

/*
 * Mxfp8VarlenMeta.from_lengths (LP-FA4 README, "MXFP8 forward and backward").
 * On entry meta->dev must point to the caller's device buffer; on return the scalar
 * fields are set and one host-to-device copy of the arrays is enqueued on `stream`.
 * Errors as for lpfa_varlen_meta_fill_host, plus LPFA_ERR_INVALID_ARG for meta->dev NULL.
 */
LPFA_API lpfa_status lpfa_varlen_meta_from_lengths(const int32_t* lengths_host, int32_t num_seqs,
                                          lpfa_varlen_meta* meta, void* stream);

/* Bytes of scale storage for one quantized tensor: total_scale_blocks * heads * 512. */
LPFA_API size_t lpfa_scale_bytes(const lpfa_varlen_meta* meta, int32_t heads);

/*
 * quantize_mxfp8_varlen (LP-FA4 README, "MXFP8 forward and backward": E4M3 payload plus
 * one E8M0 scale per 32-element block along head_dim; RCEIL default, FLOOR optional;
 * per-sequence 128-token-padded scale storage; quantization happens before the kernel).
 *
 * x          device, (T, H, 128) values of dtype `dt`; element (t, h, d) is at
 *            x + t * tok_stride + h * head_stride + d (strides in elements; d is
 *            contiguous). Values must be finite.
 * payload    device, (T, H, 128) uint8 E4M3 codes, contiguous.
 * scales     device, lpfa_scale_bytes(meta, heads) bytes. For sequence i, 128-token block b,
 *            head h the 512-byte atom at ((scale_off[i] + b) * H + h) * 512 holds the scale
 *            byte of token row r (0..127) and 32-element block kb (0..3) at
 *            (r % 32) * 16 + (r / 32) * 4 + kb. Byte = e + 127 for the power of two 2^e.
 *            Rows past the end of the sequence are written as 0x7F.
 * Rules:     RCEIL: smallest e with amax <= 448 * 2^e; FLOOR: e = floor(log2 amax) - 8;
 *            e clamped to [-127, 127]; amax == 0 gives byte 0x00. Payload is
 *            E4M3(x * 2^-e), round to nearest even, saturating to +-448, sign kept.
 * Alignment: x 16-byte aligned with tok_stride and head_stride multiples of 8 elements
 *            (bf16) or 4 elements (fp32); payload 16-byte aligned.
 * Errors:    LPFA_ERR_INVALID_ARG for NULL pointers, bad enums, head_dim != 128,
 *            heads < 1, meta without a device buffer, or misalignment.
 */
LPFA_API lpfa_status lpfa_quantize_mxfp8_varlen(const void* x, lpfa_in_dtype dt, int64_t tok_stride,
                                       int64_t head_stride, int32_t heads, int32_t head_dim,
                                       const lpfa_varlen_meta* meta, lpfa_scaling_mode mode,
                                       uint8_t* payload, uint8_t* scales, void* stream);

/*
 * The second hardware orientation of quantize_mxfp8_varlen (LP-FA4 README, "MXFP8 forward and
 * backward": Q, K and V retain both hardware orientations needed across forward and backward):
 * one E8M0 scale per 32 consecutive tokens of one (head, channel), groups aligned to the start
 * of each sequence (4 per 128-token block). Arguments, alignment, errors and the scale rules
 * are those of lpfa_quantize_mxfp8_varlen; only the blocking and the atom layout differ:
 *
 * payload    (T, H, 128) E4M3 codes, E4M3(x * 2^-e) with e the scale of the element's
 *            (32-token group, channel).
 * scales     the same storage size (lpfa_scale_bytes); the atom of (sequence i, 128-token
 *            block b, head h) at ((scale_off[i] + b) * H + h) * 512 holds the scale of channel
 *            n, token group g at byte (n % 32) * 16 + (n / 32) * 4 + g. A partial last group
 *            takes its maximum over the tokens it has; a group with no token holds 0x7F.
 *
 * This is V's layout for LPFA_PV_MXFP8 (the PV product's K dimension is the keys).
 */
LPFA_API lpfa_status lpfa_quantize_mxfp8_varlen_tokens(const void* x, lpfa_in_dtype dt, int64_t tok_stride,
                                              int64_t head_stride, int32_t heads, int32_t head_dim,
                                              const lpfa_varlen_meta* meta, lpfa_scaling_mode mode,
                                              uint8_t* payload, uint8_t* scales, void* stream);

/*
 * fa4_v_to_fp8 (FastVideo #1654: the fp8 PV mode feeds V as an unscaled E4M3 cast, with no
 * scale factors and an implicit dequant scale of 1.0).
 *
 * v          device, (tokens, H, 128) bf16 with strides as for the quantizer.
 * out        device, (tokens, H, 128) uint8 E4M3 codes, contiguous; round to nearest even,
 *            saturating to +-448, sign kept.
 * Errors:    LPFA_ERR_INVALID_ARG for NULL pointers, tokens < 1, heads < 1,
 *            head_dim != 128 or misalignment.
 */
LPFA_API lpfa_status lpfa_cast_e4m3(const void* v_bf16, int64_t tok_stride, int64_t head_stride,
                           int64_t tokens, int32_t heads, int32_t head_dim, uint8_t* out,
                           void* stream);

/*
 * MXFP8 to BF16: the exact values of a quantize_mxfp8_varlen payload (LP-FA4 README, "MXFP8
 * forward and backward": E4M3 payload times the E8M0 power of two of its 32-element block along
 * head_dim). Value (t, h, d) = E4M3(payload) * 2^e, computed in FP32 and rounded once to BF16:
 * exact whenever the product is a normal BF16 number (every scale byte >= 3, i.e. e >= -124);
 * smaller scales round the subnormal results to nearest even. These are the values that the bf16
 * PV mode multiplies (the same bits as its in-kernel conversion).
 *
 * payload    device, (T, H, 128) E4M3 codes, contiguous, 16-byte aligned.
 * scales     device, the scale storage of lpfa_quantize_mxfp8_varlen under meta.
 * out_bf16   device, (T, H, 128) bf16, contiguous, 16-byte aligned; every token row is written.
 * Errors:    LPFA_ERR_INVALID_ARG for NULL pointers, head_dim != 128, heads < 1, meta without a
 *            device buffer, or misalignment; LPFA_ERR_UNSUPPORTED off sm_100; LPFA_ERR_CUDA on
 *            launch failure.
 */
LPFA_API lpfa_status lpfa_dequantize_mxfp8_varlen(const uint8_t* payload, const uint8_t* scales,
                                         const lpfa_varlen_meta* meta, int32_t heads,
                                         int32_t head_dim, void* out_bf16, void* stream);

/*
 * mxfp8_flash_attn_varlen_forward (LP-FA4 README, "MXFP8 forward and backward": noncausal,
 * head-dim-128 MHA over packed variable-length sequences, returning out and lse), with the
 * fp8 PV mode of FastVideo #1654 and the per-tensor descales of vLLM #63232.
 *
 * q, q_sf          device, Q payload (Tq, H, 128) and its scale storage under meta_q.
 * k, k_sf          device, K payload (Tk, H, 128) and its scale storage under meta_k.
 * v, v_sf          device, V payload (Tk, H, 128). LPFA_PV_BF16: an MXFP8 payload whose scale
 *                  storage (under meta_k) is v_sf; it is dequantized exactly to BF16 and P is
 *                  rounded to BF16 for the PV product. LPFA_PV_FP8: unscaled E4M3 codes (see
 *                  lpfa_cast_e4m3), v_sf must be NULL, P is rounded to E4M3 relative to a
 *                  power-of-two running maximum. LPFA_PV_BF16_V: v points to BF16 values
 *                  (Tk, H, 128), contiguous, never quantized (LP-FA4 README: V kept in BF16);
 *                  v_sf must be NULL; P is rounded to BF16 as in LPFA_PV_BF16.
 *                  LPFA_PV_MXFP8: block-scaled MXFP8 PV; v and v_sf are V quantized in the
 *                  token orientation (lpfa_quantize_mxfp8_varlen_tokens, under meta_k), and P
 *                  is quantized to MXFP8 per 32 keys (RCEIL on each group's maximum) before a
 *                  block-scaled E4M3 x E4M3 product; O is divided by the sum of the unrounded P.
 * meta_q, meta_k   sequence i of meta_q attends to sequence i of meta_k (same num_seqs).
 * q/k/v_descale    device pointers to one float each, or NULL (per-tensor descales; see
 *                  lpfa_attn_fwd_varlen_descaled for per-head ones). NULL means exactly 1.0:
 *                  the kernel then uses the literal 1.0f on the same code path, so a descale
 *                  of 1.0 gives bit-identical output to NULL. Logits are scaled by
 *                  q_descale * k_descale / sqrt(128), O by v_descale. Values must be finite.
 * out_bf16         device, (Tq, H, 128) bf16, written for every real token row.
 * lse              device, (H, Tq) fp32, natural-log logsumexp of the scaled logits.
 * Alignment:       every tensor 16-byte aligned.
 * Errors:          LPFA_ERR_INVALID_ARG for NULL required pointers, head_dim != 128,
 *                  heads < 1, mismatched num_seqs, a bad pv_mode, or a non-NULL v_sf in fp8
 *                  or BF16-V mode (and NULL v_sf in bf16 or MXFP8 mode); LPFA_ERR_UNSUPPORTED off sm_100;
 *                  LPFA_ERR_CUDA on launch failure. A kernel that gives up on a barrier wait
 *                  records LPFA_ERR_TIMEOUT in the device status word (see below).
 */
LPFA_API lpfa_status lpfa_attn_fwd_varlen(const uint8_t* q, const uint8_t* q_sf, const uint8_t* k,
                                 const uint8_t* k_sf, const uint8_t* v, const uint8_t* v_sf,
                                 const lpfa_varlen_meta* meta_q, const lpfa_varlen_meta* meta_k,
                                 int32_t heads, int32_t head_dim, lpfa_pv_mode pv_mode,
                                 const float* q_descale, const float* k_descale,
                                 const float* v_descale, void* out_bf16, float* lse,
                                 void* stream);

/*
 * A descale tensor indexed by (sequence, head) (vLLM #63232, "Claims": calibrated per-tensor
 * scales and per-head scales keep their descale tensors; FA4's descale views are
 * (batch, kv_heads)). The value for sequence i, head h is ptr[i * seq_stride + h * head_stride]
 * (strides in elements, >= 0): per tensor (0, 0), per head (0, 1), one value per sequence and
 * head (heads, 1). ptr NULL means exactly 1.0 everywhere, the strides are then ignored. The
 * caller owns the device buffer, which must hold every index the strides reach for
 * i < num_seqs, h < heads.
 */
typedef struct {
  const float* ptr;
  int64_t seq_stride;
  int64_t head_stride;
} lpfa_descale;

/*
 * lpfa_attn_fwd_varlen with descales per (sequence, head). Arguments and behaviour as
 * lpfa_attn_fwd_varlen, except that q/k/v_descale point to lpfa_descale descriptors (host
 * memory, read before the call returns); a NULL descriptor or a NULL ptr means exactly 1.0 on
 * the same code path, so descale values of 1.0 give bit-identical output to no descale.
 * The logits of sequence i, head h are scaled by q(i,h) * k(i,h) / sqrt(128), its O rows by
 * v(i,h). Errors: as lpfa_attn_fwd_varlen, plus LPFA_ERR_INVALID_ARG for a negative stride.
 */
LPFA_API lpfa_status lpfa_attn_fwd_varlen_descaled(const uint8_t* q, const uint8_t* q_sf, const uint8_t* k,
                                          const uint8_t* k_sf, const uint8_t* v, const uint8_t* v_sf,
                                          const lpfa_varlen_meta* meta_q, const lpfa_varlen_meta* meta_k,
                                          int32_t heads, int32_t head_dim, lpfa_pv_mode pv_mode,
                                          const lpfa_descale* q_descale, const lpfa_descale* k_descale,
                                          const lpfa_descale* v_descale, void* out_bf16, float* lse,
                                          void* stream);

/*
 * Shared-query forward (LP-FA4 README, opening paragraph: the MXFP8 API covers "dense, packed
 * variable-length, and shared-query workloads"; the pages do not define the last). Reading taken:
 * one query sequence is shared by n key/value sequences, and each key/value sequence i gives its
 * own output block, O_i = attention(Q, K_i, V_i) (and LSE_i), stacked along the tokens. The kernel
 * reads the shared Q tiles for every block instead of a copy per block, longest K/V first.
 *
 * q, q_sf          device, Q payload (Lq, H, 128) and its scale storage under meta_q, which must
 *                  describe exactly one sequence of Lq tokens.
 * k, k_sf, v, v_sf as for lpfa_attn_fwd_varlen, under meta_k (n >= 1 sequences).
 * pv_mode          as for lpfa_attn_fwd_varlen.
 * q/k/v_descale    as for lpfa_attn_fwd_varlen_descaled; the sequence index is that of the
 *                  key/value sequence (0 .. n - 1).
 * out_bf16         device, (n * Lq, H, 128) bf16: rows [i * Lq, (i + 1) * Lq) are block i.
 * lse              device, (H, n * Lq) fp32, natural log, blocks laid out like out's rows.
 * Alignment:       every tensor 16-byte aligned.
 * Errors:          as for lpfa_attn_fwd_varlen, with meta_q.num_seqs != 1 (instead of a mismatch of
 *                  sequence counts) and n * Lq above INT32_MAX returning LPFA_ERR_INVALID_ARG.
 */
LPFA_API lpfa_status lpfa_attn_fwd_shared_q(const uint8_t* q, const uint8_t* q_sf, const uint8_t* k,
                                   const uint8_t* k_sf, const uint8_t* v, const uint8_t* v_sf,
                                   const lpfa_varlen_meta* meta_q, const lpfa_varlen_meta* meta_k,
                                   int32_t heads, int32_t head_dim, lpfa_pv_mode pv_mode,
                                   const lpfa_descale* q_descale, const lpfa_descale* k_descale,
                                   const lpfa_descale* v_descale, void* out_bf16, float* lse,
                                   void* stream);

/*
 * The bf16 PV mode with V converted once (LP-FA4 README, "MXFP8 forward and backward": V's
 * MXFP8 payload is dequantized exactly to BF16 for the BF16 PV product). Without a workspace the
 * attention kernel converts each 128-key V tile in shared memory every time a pair of query
 * tiles reads it; with one, lpfa_dequantize_mxfp8_varlen writes BF16 V there first and the
 * kernel reads it as BF16 V input. Both give the same bits.
 *
 * lpfa_attn_fwd_workspace_bytes returns the workspace size a call needs: total_tokens(meta_k)
 * * heads * 256 bytes for LPFA_PV_BF16, 0 for the other modes (and for invalid arguments).
 *
 * lpfa_attn_fwd_varlen_ws / lpfa_attn_fwd_shared_q_ws: arguments and behaviour of
 * lpfa_attn_fwd_varlen_descaled / lpfa_attn_fwd_shared_q, plus
 * workspace        device, 16-byte aligned, at least workspace_bytes bytes, owned by the caller;
 *                  written by the call (its contents afterwards are BF16 V) and free again once
 *                  the call's work on `stream` has finished. Ignored (may be NULL) when the mode
 *                  needs none.
 * Errors:          as those entry points, plus LPFA_ERR_INVALID_ARG in LPFA_PV_BF16 mode for a
 *                  NULL or misaligned workspace or one below lpfa_attn_fwd_workspace_bytes.
 */
LPFA_API size_t lpfa_attn_fwd_workspace_bytes(const lpfa_varlen_meta* meta_k, int32_t heads,
                                              lpfa_pv_mode pv_mode);
LPFA_API lpfa_status lpfa_attn_fwd_varlen_ws(const uint8_t* q, const uint8_t* q_sf, const uint8_t* k,
                                    const uint8_t* k_sf, const uint8_t* v, const uint8_t* v_sf,
                                    const lpfa_varlen_meta* meta_q, const lpfa_varlen_meta* meta_k,
                                    int32_t heads, int32_t head_dim, lpfa_pv_mode pv_mode,
                                    const lpfa_descale* q_descale, const lpfa_descale* k_descale,
                                    const lpfa_descale* v_descale, void* out_bf16, float* lse,
                                    void* workspace, size_t workspace_bytes, void* stream);
LPFA_API lpfa_status lpfa_attn_fwd_shared_q_ws(const uint8_t* q, const uint8_t* q_sf, const uint8_t* k,
                                      const uint8_t* k_sf, const uint8_t* v, const uint8_t* v_sf,
                                      const lpfa_varlen_meta* meta_q, const lpfa_varlen_meta* meta_k,
                                      int32_t heads, int32_t head_dim, lpfa_pv_mode pv_mode,
                                      const lpfa_descale* q_descale, const lpfa_descale* k_descale,
                                      const lpfa_descale* v_descale, void* out_bf16, float* lse,
                                      void* workspace, size_t workspace_bytes, void* stream);

/*
 * Forward without any device allocation (the pages have no counterpart; this is a library
 * convenience). Some callers cannot give the library device memory: code embedded in a host
 * application or serving runtime whose own pool owns every byte of the GPU and forbids other
 * allocations, and latency-critical paths where cudaMalloc / cudaFree (which can synchronise the
 * whole device) are not allowed. lpfa_attn_fwd_varlen_ws needs a caller workspace in bf16 PV mode;
 * this entry point takes the same arguments minus the workspace and uses a fixed scratch array
 * inside the library instead (LPFA_NOALLOC_SCRATCH_BYTES = 64 MiB of device memory, reserved on
 * every GPU where the library is loaded, until the process exits). It calls no cudaMalloc, cudaFree
 * or other allocating routine.
 *
 * Arguments, results and errors: as lpfa_attn_fwd_varlen_descaled (same bits as that call and as
 * lpfa_attn_fwd_varlen_ws). Modes other than LPFA_PV_BF16 need no scratch and take any size.
 * Limit:   in LPFA_PV_BF16 mode, total_tokens(meta_k) * heads * 256 bytes (the BF16 copy of V) must
 *          fit in the scratch, i.e. key tokens x heads <= 262144 (e.g. 16384 tokens at 16 heads);
 *          larger calls return LPFA_ERR_INVALID_ARG before any work, with the sizes in the message.
 * Set-up:  the first call on a device (with that device current) looks up the scratch array's
 *          device address (cudaGetSymbolAddress) and keeps it; make that first call before any
 *          stream capture on that device.
 * Sharing: every call on a device uses the same scratch, which keeps the last call's contents (no
 *          part of it needs to start at zero: each call writes all the scratch it reads first).
 *          Calls whose work overlaps on the GPU (different streams, or different host threads
 *          without ordering) race on it and give wrong results; order them on one stream.
 */
#define LPFA_NOALLOC_SCRATCH_BYTES (64ull << 20)
LPFA_API lpfa_status lpfa_attn_fwd_varlen_noalloc(const uint8_t* q, const uint8_t* q_sf, const uint8_t* k,
                                         const uint8_t* k_sf, const uint8_t* v, const uint8_t* v_sf,
                                         const lpfa_varlen_meta* meta_q, const lpfa_varlen_meta* meta_k,
                                         int32_t heads, int32_t head_dim, lpfa_pv_mode pv_mode,
                                         const lpfa_descale* q_descale, const lpfa_descale* k_descale,
                                         const lpfa_descale* v_descale, void* out_bf16, float* lse,
                                         void* stream);

/*
 * mxfp8_flash_attn_varlen_backward (LP-FA4 README, "MXFP8 forward and backward"): the gradients
 * of lpfa_attn_fwd_varlen's output with respect to the dequantized Q, K, V (quantization is not
 * differentiated), noncausal head-dim-128 MHA over packed variable-length sequences:
 *   P = exp(S - lse), dV = vd P^T dO, dP = vd dO V^T, D = rowsum(dO * O), dS = P * (dP - D),
 *   dQ = c dS K, dK = c dS^T Q, with S = Q K^T * c and c = qd * kd / sqrt(128).
 *
 * q, q_sf, k, k_sf, v, v_sf   MXFP8 Q, K, V with head_dim-orientation scale storage (as the
 *                  quantizer writes them; v_sf required).
 * out_bf16, dout_bf16   device, (Tq, H, 128) bf16: the forward's O and the incoming gradient.
 * lse              device, (H, Tq) fp32, the forward's natural-log LSE.
 * meta_q, meta_k, heads, head_dim   as for lpfa_attn_fwd_varlen.
 * q/k/v_descale    as for lpfa_attn_fwd_varlen_descaled (NULL descriptors or pointers: 1.0).
 * dq_bf16          device, (Tq, H, 128) bf16 output. Before dQ is written, its first Tq * H * 4
 *                  bytes hold D = rowsum(dO * O) as fp32 for the dK/dV kernel, so it must not
 *                  overlap any input.
 * dk, dv           device, (Tk, H, 128): bf16 when output_mxfp8_dkv is 0; E4M3 payloads when it
 *                  is 1, with E8M0 scales (one per 32 elements along head_dim, RCEIL) written to
 *                  dk_sf and dv_sf in the quantizer's scale storage layout under meta_k.
 * Alignment:       every tensor 16-byte aligned.
 * Errors:          LPFA_ERR_INVALID_ARG for NULL required pointers (dk_sf/dv_sf when
 *                  output_mxfp8_dkv), head_dim != 128, heads < 1, mismatched num_seqs, misalignment
 *                  or a negative descale stride; LPFA_ERR_UNSUPPORTED off sm_100; LPFA_ERR_CUDA on
 *                  launch failure; a kernel whose bounded wait runs out records LPFA_ERR_TIMEOUT.
 * The library allocates nothing; three kernels (D per row, dK/dV per key tile, dQ per query
 * tile) run on `stream`.
 */
LPFA_API lpfa_status lpfa_attn_bwd_varlen(const uint8_t* q, const uint8_t* q_sf, const uint8_t* k,
                                 const uint8_t* k_sf, const uint8_t* v, const uint8_t* v_sf,
                                 const void* out_bf16, const void* dout_bf16, const float* lse,
                                 const lpfa_varlen_meta* meta_q, const lpfa_varlen_meta* meta_k,
                                 int32_t heads, int32_t head_dim, const lpfa_descale* q_descale,
                                 const lpfa_descale* k_descale, const lpfa_descale* v_descale,
                                 void* dq_bf16, void* dk, void* dv, uint8_t* dk_sf, uint8_t* dv_sf,
                                 int32_t output_mxfp8_dkv, void* stream);

/*
 * Device status word. Kernels that bound their barrier waits record a failure code in a
 * library-owned device word instead of hanging. This call synchronizes `stream`, reads the
 * word of the current device, resets it to zero, and returns LPFA_OK, LPFA_ERR_TIMEOUT, or
 * LPFA_ERR_CUDA if the synchronization itself failed. *detail (may be NULL) receives the
 * recorded diagnostic (which wait gave up), 0 if none.
 *
 * There is one such word per device and process, shared by every kernel of this library and
 * every stream: the first failure since the last read is kept (later ones leave it alone), and
 * a read clears it. Calls that run concurrently on several streams therefore share one status;
 * the stream argument only chooses what is synchronized before the read. Callers that need a
 * status per stream must serialise the calls whose status they read.
 */
LPFA_API lpfa_status lpfa_device_status(void* stream, int32_t* detail);

/*
 * Test hook for the bounded-wait failure path (no counterpart on the pages). Same arguments
 * and behaviour as lpfa_attn_fwd_varlen, plus debug_flags: with bit 0 set, the kernel's QK
 * issuer first waits on a barrier phase that nothing completes, so its bounded wait runs out
 * (about 2 s), the kernel records LPFA_ERR_TIMEOUT in the device status word (read it with
 * lpfa_device_status) and every role exits after its in-flight copies and MMAs have landed;
 * out_bf16 and lse are then unspecified. The GPU context stays usable. debug_flags = 0 is
 * exactly lpfa_attn_fwd_varlen.
 */
LPFA_API lpfa_status lpfa_attn_fwd_varlen_debug(const uint8_t* q, const uint8_t* q_sf, const uint8_t* k,
                                       const uint8_t* k_sf, const uint8_t* v, const uint8_t* v_sf,
                                       const lpfa_varlen_meta* meta_q, const lpfa_varlen_meta* meta_k,
                                       int32_t heads, int32_t head_dim, lpfa_pv_mode pv_mode,
                                       const float* q_descale, const float* k_descale,
                                       const float* v_descale, void* out_bf16, float* lse,
                                       void* stream, int32_t debug_flags);

/*
 * Test hook for the backward's bounded-wait failure path (no counterpart on the pages). Same
 * arguments and behaviour as lpfa_attn_bwd_varlen, plus debug_flags: with bit 0 set, the MMA
 * issue warp of the dK/dV kernel first waits on a barrier phase that nothing completes, so its
 * bounded wait runs out (about 2 s per wave of CTAs), the kernel records LPFA_ERR_TIMEOUT in the
 * device status word (site 207) and every role exits after its in-flight MMAs have completed;
 * dk, dv (and their scales) are then unspecified. The dQ kernel runs normally. The GPU context
 * stays usable. Other bits are rejected with LPFA_ERR_INVALID_ARG; debug_flags = 0 is exactly
 * lpfa_attn_bwd_varlen.
 */
LPFA_API lpfa_status lpfa_attn_bwd_varlen_debug(const uint8_t* q, const uint8_t* q_sf, const uint8_t* k,
                                       const uint8_t* k_sf, const uint8_t* v, const uint8_t* v_sf,
                                       const void* out_bf16, const void* dout_bf16, const float* lse,
                                       const lpfa_varlen_meta* meta_q, const lpfa_varlen_meta* meta_k,
                                       int32_t heads, int32_t head_dim, const lpfa_descale* q_descale,
                                       const lpfa_descale* k_descale, const lpfa_descale* v_descale,
                                       void* dq_bf16, void* dk, void* dv, uint8_t* dk_sf, uint8_t* dv_sf,
                                       int32_t output_mxfp8_dkv, void* stream, int32_t debug_flags);

/* Message describing the last non-OK status returned on the calling thread ("" if none). */
LPFA_API const char* lpfa_last_error_message(void);

/* Library version string. */
LPFA_API const char* lpfa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LPFA_H */
