"""Noncausal head-dim-128 attention forward on dequantized inputs (oracle side, float64).

Plain definition (LP-FA4 README, "MXFP8 forward and backward": noncausal
head_dim-128 MHA, ``out, lse = mxfp8_flash_attn_varlen_forward(...)``):

    s_rj  = (q_r . k_j) * qd * kd / sqrt(128)      for keys j of the same sequence
    m_r   = max_j s_rj
    w_rj  = exp(s_rj - m_r),  l_r = sum_j w_rj
    O_r   = (sum_j w_rj v_j) / l_r * vd
    LSE_r = m_r + ln(l_r)                          (natural log)

Sequence i of the query metadata attends to sequence i of the key metadata
(cross attention pairs sequences by index). Descales qd, kd, vd default to
exactly 1.0 when absent (vLLM PR #63232, "Claims": a missing descale is read as
1.0). qd and kd act on the logits, vd on the output. Each is a scalar (per
tensor) or an array indexed by (sequence, head): shape (H,) for per-head scales,
(num_seqs, H) for FA4's (batch, kv_heads) descale layout, size-1 axes broadcast
(same page: calibrated per-tensor and per-head scales keep their descale
tensors). Reading: with MHA, the KV head of a query head is that head.

fp8 PV grading variant (``p_mode="fp8"``). FastVideo PR #1654 feeds PV with
plain fp8 operands but does not say how P is rounded. The reading used here,
and implemented by the CUDA kernel, rounds P to E4M3 relative to a power-of-two
reference: with t_j = s_j * log2(e) and m* = ceil(max_j t_j),

    w~_j = 2^-8 * E4M3(2^8 * 2^(t_j - m*)),
    O_r  = (sum_j w~_j v_j) / (sum_j 2^(t_j - m*)) * vd,

and LSE as in the plain definition. Because E4M3 rounding commutes with exact
power-of-two scaling outside the subnormal range, any schedule whose running
maximum is an integer in log2 units reproduces these weights.

Block-scaled MXFP8 PV variant (``p_mode="mxfp8"``; the block-scaled PV of LP-FA4, where P
and V are both MXFP8 with their 32-element blocks along the keys). Reading: P is quantized
exactly as the quantizer would quantize it, relative to any power-of-two reference:

    u_j  = 2^(t_j - m*),  32-key groups aligned to the sequence's first key,
    e_g  = RCEIL exponent of max_{j in g} u_j,
    w~_j = E4M3(u_j * 2^-e_g) * 2^e_g,
    O_r  = (sum_j w~_j v_j) / (sum_j u_j) * vd,

with V the token-orientation dequantized values; the LSE as in the plain definition. The
E8M0 scale absorbs the power of two, so the weights do not depend on m* or on a kernel's
tile schedule (outside the clamp of e to [-127, 127]).

Parity: the plain definition is pinned by closed forms (constant V, a single
key, equal logits), by a brute-force pure-Python softmax on tiny inputs, by
scipy's logsumexp, and by invariances (key permutation, packing vs separate
sequences, descale 2 == scale bytes + 1). The fp8 variant is pinned where it
reduces to the plain definition (weights that are exact E4M3 values), by its
invariance under logit shifts of k * ln 2, and by a brute-force loop that
encodes with nearest search over the E4M3 table.
"""
from __future__ import annotations

import math

import numpy as np

from . import meta as _meta
from . import mxfp8 as _mx

HEAD_DIM = 128
LOG2E = 1.0 / math.log(2.0)


def _fp8_weights(t: np.ndarray) -> np.ndarray:
    """w~ = 2^-8 * E4M3(2^8 * 2^(t - ceil(max t))) per row; also returns unrounded 2^(t - m*)."""
    mstar = np.ceil(t.max(axis=-1, keepdims=True))
    u = np.exp2(t - mstar)
    w = _mx.e4m3_decode(_mx.e4m3_encode(u * 256.0)) / 256.0
    return w, u


def descale_at(d, seq: int, head: int) -> float:
    """The descale value for (sequence, head): d is a scalar, an (H,) array, or an (S, H) array
    whose size-1 axes broadcast."""
    a = np.asarray(d, dtype=np.float64)
    if a.ndim == 0:
        return float(a)
    if a.ndim == 1:
        return float(a[head if a.shape[0] > 1 else 0])
    if a.ndim == 2:
        return float(a[seq if a.shape[0] > 1 else 0, head if a.shape[1] > 1 else 0])
    raise ValueError("a descale is a scalar, (H,) or (S, H)")


def _mx_weights(t: np.ndarray):
    """Block-scaled MXFP8 P per row (see the module docstring): (w~, u), both relative to 2^m*."""
    mstar = np.ceil(t.max(axis=-1, keepdims=True))
    u = np.exp2(t - mstar)
    R, N = u.shape
    pad = (-N) % _mx.BLOCK
    up = np.concatenate([u, np.zeros((R, pad))], axis=1).reshape(R, -1, _mx.BLOCK)
    e = _mx.e8m0_exponent(up.max(axis=2), "rceil")                 # (R, groups)
    w = _mx.e4m3_decode(_mx.e4m3_encode(up * np.ldexp(1.0, -e)[..., None])) * np.ldexp(1.0, e)[..., None]
    return w.reshape(R, -1)[:, :N], u


def attend_block(q, k, v, qd=1.0, kd=1.0, vd=1.0, p_mode: str = "exact"):
    """Attention of query rows q (R,128) over keys k, v (N,128); returns (O (R,128), LSE (R,))."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    s = (q @ k.T) * (float(qd) * float(kd) / math.sqrt(HEAD_DIM))
    m = s.max(axis=1, keepdims=True)
    w = np.exp(s - m)
    l = w.sum(axis=1)
    lse = m[:, 0] + np.log(l)
    if p_mode == "exact":
        o = (w @ v) / l[:, None] * float(vd)
    elif p_mode == "fp8":
        wq, u = _fp8_weights(s * LOG2E)
        o = (wq @ v) / u.sum(axis=1)[:, None] * float(vd)
    elif p_mode == "mxfp8":
        wq, u = _mx_weights(s * LOG2E)
        o = (wq @ v) / u.sum(axis=1)[:, None] * float(vd)
    else:
        raise ValueError("p_mode must be 'exact', 'fp8' or 'mxfp8'")
    return o, lse


def attention_fwd(qhat, khat, vhat, lengths_q, lengths_k, qd=1.0, kd=1.0, vd=1.0,
                  p_mode: str = "exact"):
    """Full varlen forward. qhat (Tq,H,128), khat/vhat (Tk,H,128) float64.

    Returns O (Tq, H, 128) float64 and LSE (H, Tq) float64.
    """
    mq = _meta.from_lengths(lengths_q)
    mk = _meta.from_lengths(lengths_k)
    if mq.num_seqs != mk.num_seqs:
        raise ValueError("query and key metadata must describe the same number of sequences")
    Tq, H, _ = qhat.shape
    out = np.zeros((Tq, H, HEAD_DIM), dtype=np.float64)
    lse = np.zeros((H, Tq), dtype=np.float64)
    for i in range(mq.num_seqs):
        q0, q1 = int(mq.cu_seqlens[i]), int(mq.cu_seqlens[i + 1])
        k0, k1 = int(mk.cu_seqlens[i]), int(mk.cu_seqlens[i + 1])
        for h in range(H):
            o, l = attend_block(qhat[q0:q1, h], khat[k0:k1, h], vhat[k0:k1, h],
                                descale_at(qd, i, h), descale_at(kd, i, h), descale_at(vd, i, h), p_mode)
            out[q0:q1, h] = o
            lse[h, q0:q1] = l
    return out, lse


def attention_rows(qhat_rows, seq_of_row, head_of_row, khat, vhat, lengths_k,
                   qd=1.0, kd=1.0, vd=1.0, p_mode: str = "exact"):
    """Attention for selected query rows only (for sampled checks at full size).

    qhat_rows (R,128) float64; seq_of_row, head_of_row (R,) ints; khat/vhat either full
    (Tk,H,128) arrays or callables ``f(seq, head) -> (N,128)`` returning one head of one
    sequence. Returns O (R,128) and LSE (R,).
    """
    mk = _meta.from_lengths(lengths_k)
    R = len(seq_of_row)
    out = np.zeros((R, HEAD_DIM), dtype=np.float64)
    lse = np.zeros(R, dtype=np.float64)
    groups = {}
    for r in range(R):
        groups.setdefault((int(seq_of_row[r]), int(head_of_row[r])), []).append(r)
    for (i, h), rows in groups.items():
        if callable(khat):
            kk, vv = khat(i, h), vhat(i, h)
        else:
            k0, k1 = int(mk.cu_seqlens[i]), int(mk.cu_seqlens[i + 1])
            kk, vv = khat[k0:k1, h], vhat[k0:k1, h]
        o, l = attend_block(np.asarray(qhat_rows)[rows], kk, vv, descale_at(qd, i, h),
                            descale_at(kd, i, h), descale_at(vd, i, h), p_mode)
        out[rows] = o
        lse[rows] = l
    return out, lse


def attention_fwd_shared_q(qhat, khat, vhat, lengths_k, qd=1.0, kd=1.0, vd=1.0, p_mode: str = "exact"):
    """Shared-query forward: one query set attends to each of several key/value sequences.

    Reading of the LP-FA4 README's "shared-query workloads" (its opening paragraph names them
    beside dense and packed variable-length ones but does not define them): the query sequence
    is shared, and key/value sequence i of the packed K/V gives its own output block,

        O_i = attention(Q, K_i, V_i),   LSE_i likewise,   i = 0 .. n - 1,

    stacked along the tokens. qhat (Lq,H,128); khat/vhat (Tk,H,128) float64; descales are
    indexed by (key/value sequence, head). Returns O (n*Lq, H, 128) and LSE (H, n*Lq).
    """
    mk = _meta.from_lengths(lengths_k)
    Lq, H, _ = qhat.shape
    n = mk.num_seqs
    out = np.zeros((n * Lq, H, HEAD_DIM), dtype=np.float64)
    lse = np.zeros((H, n * Lq), dtype=np.float64)
    for i in range(n):
        k0, k1 = int(mk.cu_seqlens[i]), int(mk.cu_seqlens[i + 1])
        for h in range(H):
            o, l = attend_block(qhat[:, h], khat[k0:k1, h], vhat[k0:k1, h],
                                descale_at(qd, i, h), descale_at(kd, i, h), descale_at(vd, i, h), p_mode)
            out[i * Lq:(i + 1) * Lq, h] = o
            lse[h, i * Lq:(i + 1) * Lq] = l
    return out, lse
