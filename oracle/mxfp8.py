"""MXFP8 codecs and quantizer (oracle side, exact arithmetic in float64).

What the pages fix (LP-FA4 README, "MXFP8 forward and backward"):
* the payload is E4M3 with one E8M0 scale per 32-element block along head_dim;
* RCEIL scaling is the default ("Quack 0.6.2's RCEIL"), FLOOR is optional;
* every sequence gets its own scale storage padded to 128 tokens.
FastVideo PR #1654 (description): the fp8 PV mode feeds V as an unscaled E4M3
cast, with no scale factors and an implicit dequant scale of 1.0.

Readings taken where the pages are silent:
* E4M3 is the OCP "fn" variant: bias 7, no infinities, 0x7F/0xFF are NaN,
  largest finite 448, smallest normal 2^-6, subnormals k * 2^-9.
* Encoding rounds the exact value to the nearest E4M3 value, ties to the even
  code, and saturates magnitudes above 448 to 448 (``satfinite``). The sign is
  kept, so negative values that round to zero give 0x80.
* E8M0 stores a power of two 2^e as the byte e + 127, with e clamped to
  [-127, 127]; 0xFF is never produced.
* RCEIL: e is the smallest integer with amax <= 448 * 2^e.
* FLOOR: e = floor(log2 amax) - 8 (the E4M3 largest exponent is 8); scaled
  values in (448, 512) saturate to 448.
* amax = 0: e = -127 (byte 0x00) and the payload is +-0.
* Payload = E4M3(x * 2^-e), one rounding from the exact product.
* Scale storage (head_dim orientation): for sequence i, 128-token block b, head h, the 512-byte atom at
  ``((scale_off[i] + b) * H + h) * 512``; inside it the 4 scales of token row r
  (0 <= r < 128) sit at ``(r % 32) * 16 + (r // 32) * 4 + kb``, kb = 0..3 the
  32-element block index along head_dim. Rows past the sequence end hold 0x7F
  (scale 1.0). This is the 32 x 4 x 4 atom the block-scaled tensor-core MMA
  reads its scale factors in.

The token orientation (``quantize_mxfp8_varlen_tokens``) puts the 32-element blocks along
the token axis instead (see its docstring).

Parity: the codecs are pinned by exhaustive checks against brute-force nearest
search over all 256 codes and by hand-picked values; the scale rules by
brute-force search over all exponents; the quantizer by its round trip and by
the invariance of the payload under power-of-two rescaling of the input; the token
orientation by its identity with the head_dim orientation of the transposed 128 x 128 blocks.
"""
from __future__ import annotations

import numpy as np

from . import meta as _meta

E4M3_MAX = 448.0
HEAD_DIM = 128
BLOCK = 32
ATOM_BYTES = 512


def e4m3_value(code: int) -> float:
    """Value of one E4M3 ("fn") code, by the format definition."""
    code = int(code) & 0xFF
    sign = -1.0 if (code >> 7) & 1 else 1.0
    exp_field = (code >> 3) & 0xF
    mant = code & 0x7
    if exp_field == 0xF and mant == 0x7:
        return float("nan")
    if exp_field == 0:
        return sign * (mant / 8.0) * 2.0 ** -6
    return sign * (1.0 + mant / 8.0) * 2.0 ** (exp_field - 7)


def e4m3_decode_table() -> np.ndarray:
    """All 256 E4M3 values as float64 (NaN for 0x7F and 0xFF)."""
    return np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)


_DECODE = e4m3_decode_table()


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    return _DECODE[np.asarray(codes, dtype=np.uint8)]


def e4m3_encode(x) -> np.ndarray:
    """Round-to-nearest-even, saturating encode of finite float64 values to E4M3 codes."""
    x = np.asarray(x, dtype=np.float64)
    neg = np.signbit(x)
    a = np.abs(x)
    # Spacing of E4M3 values around a: 2^(E-3) in binade [2^E, 2^(E+1)) for E >= -6,
    # and the fixed subnormal spacing 2^-9 below 2^-6.
    _, ex = np.frexp(a)                      # a = m * 2^ex, m in [0.5, 1)
    binade = np.maximum(ex - 1, -6)
    quantum = np.ldexp(1.0, binade - 3)
    q = np.rint(a / quantum) * quantum       # exact; np.rint rounds half to even
    q = np.minimum(q, E4M3_MAX)              # satfinite
    # Encode the (now representable) magnitude.
    _, eq = np.frexp(q)
    qexp = eq - 1
    normal = q >= 2.0 ** -6
    exp_field = np.where(normal, qexp + 7, 0)
    safe_exp = np.where(normal, qexp, 0)
    mant = np.where(normal, (q / np.ldexp(1.0, safe_exp) - 1.0) * 8.0, q / 2.0 ** -9)
    code = (neg.astype(np.int64) << 7) | (exp_field.astype(np.int64) << 3) | mant.astype(np.int64)
    return code.astype(np.uint8)


def e8m0_exponent(amax, mode: str = "rceil") -> np.ndarray:
    """Scale exponent e (int64) for block maxima ``amax`` >= 0 under RCEIL or FLOOR."""
    amax = np.asarray(amax, dtype=np.float64)
    if mode not in ("rceil", "floor"):
        raise ValueError("scaling mode must be 'rceil' or 'floor'")
    _, ex = np.frexp(amax)
    binade = ex - 1                          # amax in [2^binade, 2^(binade+1))
    if mode == "floor":
        e = binade - 8
    else:
        # 448 * 2^(binade-8) = 1.75 * 2^binade: the smallest candidate that can cover amax.
        lo = binade - 8
        fits = amax <= E4M3_MAX * np.ldexp(1.0, lo)
        e = np.where(fits, lo, lo + 1)
    e = np.clip(e, -127, 127)
    e = np.where(amax == 0.0, -127, e)
    return e.astype(np.int64)


def atom_offset(scale_block: int, head: int, heads: int, row: int, kb: int) -> int:
    """Byte offset of one scale in the padded scale storage."""
    return ((scale_block * heads + head) * ATOM_BYTES
            + (row % 32) * 16 + (row // 32) * 4 + kb)


def quantize_mxfp8_varlen(x, lengths, mode: str = "rceil"):
    """Quantize packed (T, H, 128) values to (payload u8 (T,H,128), scales u8 (blocks*H*512,))."""
    x = np.asarray(x, dtype=np.float64)
    T, H, D = x.shape
    if D != HEAD_DIM:
        raise ValueError("head_dim must be 128")
    m = _meta.from_lengths(lengths)
    if m.total_tokens != T:
        raise ValueError("tensor token count does not match the lengths")
    blocks = x.reshape(T, H, D // BLOCK, BLOCK)
    amax = np.abs(blocks).max(axis=3)                     # (T, H, 4)
    e = e8m0_exponent(amax, mode)                         # (T, H, 4)
    scaled = blocks * np.ldexp(1.0, -e)[..., None]        # exact in float64
    payload = e4m3_encode(scaled).reshape(T, H, D)

    scales = np.full(m.total_scale_blocks * H * ATOM_BYTES, 0x7F, dtype=np.uint8)
    for i in range(m.num_seqs):
        n = int(m.lengths[i])
        tok = np.arange(n)
        blk = m.scale_off[i] + tok // 128
        row = tok % 128
        for h in range(H):
            base = (blk * H + h) * ATOM_BYTES + (row % 32) * 16 + (row // 32) * 4
            for kb in range(4):
                scales[base + kb] = (e[m.cu_seqlens[i] + tok, h, kb] + 127).astype(np.uint8)
    return payload, scales


def scale_exponents(scales, lengths, heads: int) -> np.ndarray:
    """Read the logical (T, H, 4) scale exponents back out of the padded storage."""
    m = _meta.from_lengths(lengths)
    scales = np.asarray(scales, dtype=np.uint8)
    out = np.empty((m.total_tokens, heads, 4), dtype=np.int64)
    for i in range(m.num_seqs):
        n = int(m.lengths[i])
        tok = np.arange(n)
        blk = m.scale_off[i] + tok // 128
        row = tok % 128
        for h in range(heads):
            base = (blk * heads + h) * ATOM_BYTES + (row % 32) * 16 + (row // 32) * 4
            for kb in range(4):
                out[m.cu_seqlens[i] + tok, h, kb] = scales[base + kb].astype(np.int64) - 127
    return out


def dequantize_mxfp8(payload, scales, lengths, heads: int) -> np.ndarray:
    """x_hat = E4M3 value * 2^(byte - 127), exact in float64; shape (T, H, 128)."""
    payload = np.asarray(payload, dtype=np.uint8)
    T = payload.shape[0]
    e = scale_exponents(scales, lengths, heads)            # (T, H, 4)
    vals = e4m3_decode(payload).reshape(T, heads, 4, BLOCK)
    return (vals * np.ldexp(1.0, e)[..., None]).reshape(T, heads, HEAD_DIM)


def quantize_mxfp8_varlen_tokens(x, lengths, mode: str = "rceil"):
    """Token orientation: one E8M0 scale per 32 consecutive tokens of one (head, channel).

    LP-FA4 README ("MXFP8 forward and backward"): Q, K and V keep both hardware orientations
    needed across forward and backward; this is the second one, with the 32-element blocks along
    the token axis, as the PV product (K = keys) and the backward's transposed products read
    them. Readings taken where the pages are silent: the 32-token groups are aligned to the start of each sequence,
    4 per 128-token block; a group's amax is taken over the tokens the sequence has (a partial
    last group is not padded with data); a group with no token of the sequence holds 0x7F.
    Scale storage: the 512-byte atom of (sequence i, 128-token block b, head h) at
    ``((scale_off[i] + b) * H + h) * 512`` as in the head_dim orientation, with channel n and
    token group g at ``(n % 32) * 16 + (n // 32) * 4 + g``.
    Returns (payload u8 (T, H, 128), scales u8 (blocks * H * 512,)).
    """
    x = np.asarray(x, dtype=np.float64)
    T, H, D = x.shape
    if D != HEAD_DIM:
        raise ValueError("head_dim must be 128")
    m = _meta.from_lengths(lengths)
    if m.total_tokens != T:
        raise ValueError("tensor token count does not match the lengths")
    payload = np.empty((T, H, D), dtype=np.uint8)
    scales = np.full(m.total_scale_blocks * H * ATOM_BYTES, 0x7F, dtype=np.uint8)
    chan = np.arange(HEAD_DIM)
    for i in range(m.num_seqs):
        c0, n = int(m.cu_seqlens[i]), int(m.lengths[i])
        for g0 in range(0, n, BLOCK):
            g1 = min(n, g0 + BLOCK)
            blk = x[c0 + g0:c0 + g1]                          # (tokens in group, H, 128)
            e = e8m0_exponent(np.abs(blk).max(axis=0), mode)  # (H, 128)
            payload[c0 + g0:c0 + g1] = e4m3_encode(blk * np.ldexp(1.0, -e)[None])
            b, g = g0 // 128, (g0 % 128) // BLOCK
            for h in range(H):
                base = ((m.scale_off[i] + b) * H + h) * ATOM_BYTES
                scales[base + (chan % 32) * 16 + (chan // 32) * 4 + g] = (e[h] + 127).astype(np.uint8)
    return payload, scales


def dequantize_mxfp8_tokens(payload, scales, lengths, heads: int) -> np.ndarray:
    """x_hat of the token orientation: E4M3 value * 2^(byte - 127) of its (token group, channel)."""
    payload = np.asarray(payload, dtype=np.uint8)
    scales = np.asarray(scales, dtype=np.uint8)
    m = _meta.from_lengths(lengths)
    out = np.empty(payload.shape, dtype=np.float64)
    chan = np.arange(HEAD_DIM)
    for i in range(m.num_seqs):
        c0, n = int(m.cu_seqlens[i]), int(m.lengths[i])
        for tok in range(0, n, BLOCK):
            t1 = min(n, tok + BLOCK)
            b, g = tok // 128, (tok % 128) // BLOCK
            for h in range(heads):
                base = ((m.scale_off[i] + b) * heads + h) * ATOM_BYTES
                e = scales[base + (chan % 32) * 16 + (chan // 32) * 4 + g].astype(np.int64) - 127
                out[c0 + tok:c0 + t1, h] = e4m3_decode(payload[c0 + tok:c0 + t1, h]) * np.ldexp(1.0, e)[None]
    return out


def cast_e4m3(v) -> np.ndarray:
    """Unscaled E4M3 cast used by the fp8 PV mode (no scale factors)."""
    return e4m3_encode(np.asarray(v, dtype=np.float64))


def quantize_rows(x_rows, mode: str = "rceil"):
    """Quantize standalone 128-element rows: returns (payload (R,128) u8, exponents (R,4))."""
    x_rows = np.asarray(x_rows, dtype=np.float64)
    R = x_rows.shape[0]
    blocks = x_rows.reshape(R, 4, BLOCK)
    e = e8m0_exponent(np.abs(blocks).max(axis=2), mode)
    payload = e4m3_encode(blocks * np.ldexp(1.0, -e)[..., None]).reshape(R, HEAD_DIM)
    return payload, e
