"""Noncausal head-dim-128 attention backward on dequantized inputs (oracle side, float64).

Test infrastructure: only tests/, __graft_entry__.smoke() and bench.py's CPU legs use oracle/.

LP-FA4 README, "MXFP8 forward and backward": ``mxfp8_flash_attn_varlen_backward(q_mx, k_mx,
v_mx, out, dout, lse, meta_q, meta_k, output_mxfp8_dkv=True)`` returns dQ in BF16 and dK, dV as
E4M3 payloads with E8M0 scales, one scale per 32-element block; without the option it returns
three BF16 gradients.

Plain definition: the gradients of the forward's definition (oracle/attention.py) with respect
to the dequantized inputs, for one (sequence, head) with query rows r and keys j:

    s_rj  = (q_r . k_j) * c,        c = qd * kd / sqrt(128)
    p_rj  = exp(s_rj - lse_r)       (lse as the forward returned it)
    dV_j  = vd * sum_r p_rj dO_r
    dP_rj = vd * (dO_r . v_j)
    D_r   = dO_r . O_r              (O as the forward returned it)
    dS_rj = p_rj * (dP_rj - D_r)
    dQ_r  = c * sum_j dS_rj k_j,    dK_j = c * sum_r dS_rj q_r

Readings taken where the pages are silent: quantization is not differentiated (the gradients are those of the
dequantized inputs, the straight-through reading); MXFP8 dK and dV use the head_dim orientation
(one scale per 32 elements along head_dim of a token row, as the forward's inputs) and RCEIL
(the README's default scaling).

Parity: pinned by central finite differences of the forward oracle on small inputs (with
descales), by closed forms (a single key: dQ = dK = 0 and dV = vd * sum of dO; p summing to one
makes the dS rows sum to zero), by D_r = sum_j p_rj dP_rj when O is exact, and by packing
several sequences against running them one by one.
"""
from __future__ import annotations

import math

import numpy as np

from . import meta as _meta
from . import mxfp8 as _mx

HEAD_DIM = 128


def attend_block_backward(q, k, v, o, do, lse, qd=1.0, kd=1.0, vd=1.0):
    """Gradients (dQ (R,128), dK (N,128), dV (N,128)) of one (sequence, head)."""
    q, k, v, o, do = (np.asarray(a, dtype=np.float64) for a in (q, k, v, o, do))
    lse = np.asarray(lse, dtype=np.float64)
    c = float(qd) * float(kd) / math.sqrt(HEAD_DIM)
    s = (q @ k.T) * c
    p = np.exp(s - lse[:, None])
    dv = float(vd) * (p.T @ do)
    dp = float(vd) * (do @ v.T)
    d = np.sum(do * o, axis=1)
    ds = p * (dp - d[:, None])
    dq = c * (ds @ k)
    dk = c * (ds.T @ q)
    return dq, dk, dv


def attention_bwd(qhat, khat, vhat, o, do, lse, lengths_q, lengths_k, qd=1.0, kd=1.0, vd=1.0):
    """Full varlen backward. qhat/o/do (Tq,H,128), khat/vhat (Tk,H,128), lse (H,Tq).

    Descales follow the forward's rule (oracle/attention.py: a scalar, (H,) or (S, H)).
    Returns dQ (Tq,H,128), dK (Tk,H,128), dV (Tk,H,128), float64.
    """
    from .attention import descale_at

    mq = _meta.from_lengths(lengths_q)
    mk = _meta.from_lengths(lengths_k)
    if mq.num_seqs != mk.num_seqs:
        raise ValueError("query and key metadata must describe the same number of sequences")
    Tq, H, _ = np.shape(qhat)
    Tk = np.shape(khat)[0]
    dq = np.zeros((Tq, H, HEAD_DIM))
    dk = np.zeros((Tk, H, HEAD_DIM))
    dv = np.zeros((Tk, H, HEAD_DIM))
    for i in range(mq.num_seqs):
        q0, q1 = int(mq.cu_seqlens[i]), int(mq.cu_seqlens[i + 1])
        k0, k1 = int(mk.cu_seqlens[i]), int(mk.cu_seqlens[i + 1])
        for h in range(H):
            a, b, cc = attend_block_backward(qhat[q0:q1, h], khat[k0:k1, h], vhat[k0:k1, h], o[q0:q1, h],
                                             do[q0:q1, h], lse[h, q0:q1], descale_at(qd, i, h),
                                             descale_at(kd, i, h), descale_at(vd, i, h))
            dq[q0:q1, h] = a
            dk[k0:k1, h] = b
            dv[k0:k1, h] = cc
    return dq, dk, dv


def quantize_dkv(dk, dv, lengths_k, mode: str = "rceil"):
    """output_mxfp8_dkv: dK and dV as MXFP8 in the head_dim orientation (payload, scales) each."""
    return _mx.quantize_mxfp8_varlen(dk, lengths_k, mode), _mx.quantize_mxfp8_varlen(dv, lengths_k, mode)


def attend_block_backward_sampled(q, k, v, o, do, lse, key_idx, row_idx, qd=1.0, kd=1.0, vd=1.0):
    """Selected gradient rows of one (sequence, head), each from the same definition as
    attend_block_backward, without forming the whole score matrix: dK and dV for the keys
    key_idx (each needs one column of S over all query rows), dQ for the query rows row_idx (each
    needs one row of S over all keys). Returns (dQ[row_idx], dK[key_idx], dV[key_idx])."""
    q, k, v, o, do = (np.asarray(a, dtype=np.float64) for a in (q, k, v, o, do))
    lse = np.asarray(lse, dtype=np.float64)
    key_idx = np.asarray(key_idx, dtype=np.int64)
    row_idx = np.asarray(row_idx, dtype=np.int64)
    c = float(qd) * float(kd) / math.sqrt(HEAD_DIM)
    d = np.sum(do * o, axis=1)
    # columns j of S, P, dP, dS over every query row
    p_c = np.exp((q @ k[key_idx].T) * c - lse[:, None])
    ds_c = p_c * (float(vd) * (do @ v[key_idx].T) - d[:, None])
    dv = float(vd) * (p_c.T @ do)
    dk = c * (ds_c.T @ q)
    # rows r of S, P, dP, dS over every key
    p_r = np.exp((q[row_idx] @ k.T) * c - lse[row_idx, None])
    ds_r = p_r * (float(vd) * (do[row_idx] @ v.T) - d[row_idx, None])
    dq = c * (ds_r @ k)
    return dq, dk, dv
