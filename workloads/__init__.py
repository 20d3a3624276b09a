"""Seeded synthetic workloads for the MXFP8 attention forward path.

This module draws inputs only: sequence lengths, Q/K/V values already rounded to
the input dtype, and outlier channels. It contains none of the method's
arithmetic (no quantization, no scale rule, no softmax), so both the CUDA path
and the CPU oracle may take their inputs from here.

Shapes and value distributions follow the workloads the method's pages describe:

* LP-FA4 README, section "MXFP8 forward and backward": packed
  ``(tokens, heads, 128)`` BF16 or FP32 tensors, one length per sequence,
  dense attention expressed as uniform packed offsets.
* FastVideo PR #1654 ("fp8 PV mode for the FA4-FP4 attention path"): V fed to
  the kernel as an unscaled E4M3 cast of a BF16 tensor.

Random values come from numpy's PCG64 generator (``standard_normal`` in
float32), seeded by ``(seed, workload index, stream)``; BF16 inputs are the
float32 draws rounded to nearest-even BF16. Every array is returned as float32
holding values exactly representable in the declared input dtype, plus the
raw uint16 bit pattern for BF16 uploads.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional

import numpy as np

HEAD_DIM = 128

# Stream ids used to derive independent generators per drawn quantity.
_STREAM_LEN_Q, _STREAM_LEN_K, _STREAM_Q, _STREAM_K, _STREAM_V = 1, 2, 3, 4, 5
_STREAM_OUT_Q, _STREAM_OUT_K, _STREAM_OUT_V = 6, 7, 8


@dataclasses.dataclass(frozen=True)
class Workload:
    """A named, fully specified synthetic workload."""

    name: str
    index: int                    # stable id mixed into the seed
    heads: int
    in_dtype: str                 # "bf16" or "fp32" (Q, K and the quantized V)
    pv_mode: str                  # "bf16", "fp8", "bf16v" (BF16 V input, bf16 PV) or "mxfp8" (block-scaled PV)
    scaling_mode: str = "rceil"   # "rceil" or "floor"
    num_seqs: int = 1
    len_q: Optional[int] = None   # fixed length, or None for drawn lengths
    len_k: Optional[int] = None
    range_q: Optional[tuple] = None  # inclusive (lo, hi) when lengths are drawn
    range_k: Optional[tuple] = None
    cross: bool = False           # separate K lengths (cross attention)
    v_gain: float = 1.0           # V = bf16(N(0,1)) * v_gain (exact power of two)
    outlier_frac: float = 0.0     # fraction of (head, channel) pairs scaled
    outlier_gain: float = 1.0
    shared_q: bool = False        # one query sequence (len_q) shared by num_seqs K/V sequences
    description: str = ""


# The five workloads the method is evaluated on, plus the LP-FA4 README's bundled
# benchmark shape (section "Benchmark reproduction": batch 8, 2048 x 2048, 16 heads).
WORKLOADS: Dict[str, Workload] = {}


def _add(w: Workload) -> None:
    WORKLOADS[w.name] = w


_add(Workload("single_s256_h2", 0, heads=2, in_dtype="bf16", pv_mode="bf16",
              num_seqs=1, len_q=256, len_k=256,
              description="1 sequence, 256 queries x 256 keys, 2 heads, bf16 N(0,1), RCEIL, bf16 PV"))
_add(Workload("dense_4x2048_h16", 1, heads=16, in_dtype="bf16", pv_mode="bf16",
              num_seqs=4, len_q=2048, len_k=2048,
              description="4 x 2048 uniform packed offsets, 16 heads, bf16 N(0,1), RCEIL, bf16 PV"))
_add(Workload("varlen16_fp32_h16", 2, heads=16, in_dtype="fp32", pv_mode="bf16",
              num_seqs=16, range_q=(128, 8192),
              description="16 sequences, lengths U{128..8192}, 16 heads, fp32 N(0,1), RCEIL, bf16 PV"))
_add(Workload("video_s32768_h24_fp8pv", 3, heads=24, in_dtype="bf16", pv_mode="fp8",
              num_seqs=1, len_q=32768, len_k=32768, v_gain=2.0,
              description="batch 1, 32768 tokens, 24 heads; Q/K bf16 N(0,1) MXFP8 RCEIL; "
                          "V = E4M3(bf16(N(0,1))*2), fp8 PV"))
_add(Workload("cross_varlen_outliers_h32", 4, heads=32, in_dtype="bf16", pv_mode="bf16",
              num_seqs=8, range_q=(256, 1024), range_k=(4096, 32768), cross=True,
              outlier_frac=0.01, outlier_gain=64.0,
              description="8 sequences, sq U{256..1024}, sk U{4096..32768}, 32 heads, bf16 N(0,1) "
                          "with 1% of (head, channel) pairs x64, RCEIL, bf16 PV"))
_add(Workload("lpfa4_bundled_8x2048_h16", 5, heads=16, in_dtype="bf16", pv_mode="bf16",
              num_seqs=8, len_q=2048, len_k=2048,
              description="LP-FA4 bundled benchmark shape: 8 x 2048, 16 heads, RCEIL"))

_add(Workload("dense_4x2048_h16_bf16v", 6, heads=16, in_dtype="bf16", pv_mode="bf16v",
              num_seqs=4, len_q=2048, len_k=2048,
              description="4 x 2048 uniform packed offsets, 16 heads, bf16 N(0,1); Q/K MXFP8 RCEIL, "
                          "V kept in BF16, bf16 PV"))

_add(Workload("dense_4x2048_h16_mxpv", 7, heads=16, in_dtype="bf16", pv_mode="mxfp8",
              num_seqs=4, len_q=2048, len_k=2048,
              description="4 x 2048 uniform packed offsets, 16 heads, bf16 N(0,1); Q/K MXFP8 RCEIL, V MXFP8 "
                          "in the token orientation, block-scaled MXFP8 PV"))
_add(Workload("video_s32768_h24_mxpv", 8, heads=24, in_dtype="bf16", pv_mode="mxfp8",
              num_seqs=1, len_q=32768, len_k=32768,
              description="batch 1, 32768 tokens, 24 heads; Q/K bf16 N(0,1) MXFP8 RCEIL; V bf16 N(0,1) MXFP8 "
                          "in the token orientation, block-scaled MXFP8 PV"))

# Shared-query workload (LP-FA4 README, opening paragraph: "shared-query workloads", not defined
# there): one query sequence of 1024 tokens attending to each of 8 key/value sequences with
# lengths U{2048..16384}.
_add(Workload("shared_q1024_kv8_h16", 9, heads=16, in_dtype="bf16", pv_mode="bf16",
              num_seqs=8, len_q=1024, range_k=(2048, 16384), cross=True, shared_q=True,
              description="shared query set: 1 x 1024 queries against 8 K/V sequences, sk U{2048..16384}, "
                          "16 heads, bf16 N(0,1), RCEIL, bf16 PV"))

# The five evaluation workloads in order (the others are extra benchmark rows).
EVAL_ORDER: List[str] = [
    "single_s256_h2",
    "dense_4x2048_h16",
    "varlen16_fp32_h16",
    "video_s32768_h24_fp8pv",
    "cross_varlen_outliers_h32",
]


def _rng(seed: int, w: Workload, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, w.index, stream])))


def lengths(w: Workload, seed: int = 0):
    """Return (lengths_q, lengths_k) as int32 arrays, drawn when the workload says so."""
    if w.shared_q:
        lq = np.array([w.len_q], dtype=np.int32)
    elif w.len_q is not None:
        lq = np.full(w.num_seqs, w.len_q, dtype=np.int32)
    else:
        lo, hi = w.range_q
        lq = _rng(seed, w, _STREAM_LEN_Q).integers(lo, hi + 1, size=w.num_seqs).astype(np.int32)
    if w.cross:
        if w.len_k is not None:
            lk = np.full(w.num_seqs, w.len_k, dtype=np.int32)
        else:
            lo, hi = w.range_k
            lk = _rng(seed, w, _STREAM_LEN_K).integers(lo, hi + 1, size=w.num_seqs).astype(np.int32)
    else:
        lk = lq.copy()
    return lq, lk


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest-even BF16, returned as float32 (finite inputs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> 16) & np.uint32(1)) + np.uint32(0x7FFF)
    r = ((u + bias) & np.uint32(0xFFFF0000)).astype(np.uint32)
    return r.view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """uint16 bit patterns of float32 values that are exactly BF16."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    if np.any(u & np.uint32(0xFFFF)):
        raise ValueError("values are not exactly representable in bf16")
    return (u >> 16).astype(np.uint16)


def _normal(seed: int, w: Workload, stream: int, shape) -> np.ndarray:
    out = np.empty(shape, dtype=np.float32)
    _rng(seed, w, stream).standard_normal(size=shape, dtype=np.float32, out=out)
    return out


def _outlier_pairs(seed: int, w: Workload, stream: int) -> np.ndarray:
    """Indices into heads*128 of the (head, channel) pairs that get the outlier gain."""
    total = w.heads * HEAD_DIM
    count = int(round(w.outlier_frac * total))
    return _rng(seed, w, stream).choice(total, size=count, replace=False)


def make_tensor(w: Workload, which: str, seed: int = 0, tokens: Optional[int] = None) -> np.ndarray:
    """Draw one of "q", "k", "v" as float32 (tokens, heads, 128), exact in the input dtype.

    V of an fp8-PV workload is BF16 times ``v_gain`` (the tensor the E4M3 cast reads).
    """
    lq, lk = lengths(w, seed)
    if tokens is None:
        tokens = int(lq.sum()) if which == "q" else int(lk.sum())
    stream = {"q": _STREAM_Q, "k": _STREAM_K, "v": _STREAM_V}[which]
    x = _normal(seed, w, stream, (tokens, w.heads, HEAD_DIM))
    dtype = "bf16" if (which == "v" and w.pv_mode == "fp8") else w.in_dtype
    if dtype == "bf16":
        x = round_to_bf16(x)
    if which == "v" and w.v_gain != 1.0:
        x *= np.float32(w.v_gain)
    if w.outlier_frac > 0.0:
        ostream = {"q": _STREAM_OUT_Q, "k": _STREAM_OUT_K, "v": _STREAM_OUT_V}[which]
        pairs = _outlier_pairs(seed, w, ostream)
        flat = x.reshape(tokens, w.heads * HEAD_DIM)
        flat[:, pairs] *= np.float32(w.outlier_gain)
    return x


def outlier_scale(w: Workload, which: str, seed: int = 0) -> np.ndarray:
    """(heads, 128) float32: the outlier gain on the (head, channel) pairs ``make_tensor`` scales
    for this tensor, 1 elsewhere."""
    s = np.ones(w.heads * HEAD_DIM, dtype=np.float32)
    if w.outlier_frac > 0.0:
        ostream = {"q": _STREAM_OUT_Q, "k": _STREAM_OUT_K, "v": _STREAM_OUT_V}[which]
        s[_outlier_pairs(seed, w, ostream)] = np.float32(w.outlier_gain)
    return s.reshape(w.heads, HEAD_DIM)


def tensor_dtype(w: Workload, which: str) -> str:
    """Input dtype of the tensor as handed to the library ("bf16" or "fp32")."""
    if which == "v" and w.pv_mode == "fp8":
        return "bf16"
    return w.in_dtype


def to_torch(x: np.ndarray, dtype: str, device="cuda"):
    """Upload a float32 array to a torch device tensor as bf16 (values must be exact) or fp32."""
    import torch

    if dtype == "bf16":
        return torch.from_numpy(bf16_bits(x).view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(device)


def small_random(seed: int, lengths_q, lengths_k, heads: int, scale: float = 1.0,
                 dtype: str = "bf16"):
    """Free-form seeded Q/K/V for edge-case tests (ragged lengths, few heads)."""
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 1000])))
    tq, tk = int(np.sum(lengths_q)), int(np.sum(lengths_k))
    out = []
    for t in (tq, tk, tk):
        x = (g.standard_normal((t, heads, HEAD_DIM), dtype=np.float32) * np.float32(scale))
        out.append(round_to_bf16(x) if dtype == "bf16" else x)
    return tuple(out)
