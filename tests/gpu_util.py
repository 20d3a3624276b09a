"""Helpers for the GPU parity tests: upload seeded inputs, run the library, run the oracle.

The library side and the oracle side start from the same seeded float32 arrays (exact in
their input dtype) and share nothing else.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import workloads as wl
from oracle import attention as oatt
from oracle import backward as obwd
from oracle import meta as ometa
from oracle import mxfp8 as omx

# Tolerances fixed for the attention output (O max-abs / rel-L2 against the fp64 oracle
# before BF16 rounding, LSE max-abs).
O_MAX_ABS = 2e-2
O_REL_L2 = 1e-2
LSE_MAX_ABS = 1e-3


def to_device(x: np.ndarray, dtype: str, device="cuda") -> torch.Tensor:
    """Upload a float32 array as bf16 (exact values required) or fp32."""
    return wl.to_torch(x, dtype, device)


def gpu_quantize(lp, x: np.ndarray, dtype: str, meta, mode="rceil"):
    xd = to_device(x, dtype)
    payload, scales = lp.lpfa_quantize_mxfp8_varlen(xd, meta, scaling_mode=mode)
    return payload, scales


def compare_attention(o_gpu: torch.Tensor, lse_gpu: torch.Tensor, o_ref: np.ndarray, lse_ref: np.ndarray,
                      o_scale: np.ndarray = None):
    """Return (max_abs_O, rel_l2_O, max_abs_LSE) of the GPU result against the oracle.

    o_scale (broadcastable to O): the input scale of V's (head, channel) pairs where a workload
    plants deliberate outliers, or the magnitude of a per-head v descale. The max-abs bound is
    stated for unit-scale data, so the O error of each channel is divided by that channel's
    scale before the maximum is taken (O in a channel scaled x64 is x64 larger, and so are its
    BF16 rounding and every other error). rel-L2 and LSE are unaffected.
    """
    o = o_gpu.float().cpu().numpy().astype(np.float64)
    l = lse_gpu.float().cpu().numpy().astype(np.float64)
    d = o - o_ref
    dn = d if o_scale is None else d / np.asarray(o_scale, dtype=np.float64)
    max_abs = float(np.max(np.abs(dn))) if d.size else 0.0
    rel = float(np.linalg.norm(d) / max(np.linalg.norm(o_ref), 1e-300))
    lmax = float(np.max(np.abs(l - lse_ref))) if l.size else 0.0
    return max_abs, rel, lmax


def assert_within(stats, label=""):
    max_abs, rel, lmax = stats
    msg = f"{label}: O max-abs {max_abs:.3e}, O rel-L2 {rel:.3e}, LSE max-abs {lmax:.3e}"
    assert max_abs <= O_MAX_ABS and rel <= O_REL_L2 and lmax <= LSE_MAX_ABS, msg
    return msg


def _descale_tensor(x):
    """None, a float (one-element tensor), a numpy array (same shape) or a torch tensor (as is)."""
    if x is None or isinstance(x, torch.Tensor):
        return x
    if np.ndim(x) == 0:
        return torch.tensor([float(x)], dtype=torch.float32, device="cuda")
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to("cuda")


def run_path(lp, q, k, v, lens_q, lens_k, heads, in_dtype="bf16", pv_mode="bf16", mode="rceil",
             descales=(None, None, None), workspace=True):
    """Library path: metadata, quantize Q/K (and V in bf16 PV mode) or cast V, attention.
    workspace=False runs the bf16 PV mode with V converted inside the attention kernel."""
    mq = lp.lpfa_varlen_meta_from_lengths(lens_q)
    mk = lp.lpfa_varlen_meta_from_lengths(lens_k)
    qp, qs = gpu_quantize(lp, q, in_dtype, mq, mode)
    kp, ks = gpu_quantize(lp, k, in_dtype, mk, mode)
    if pv_mode == "fp8":
        vp, vs = lp.lpfa_cast_e4m3(to_device(v, "bf16")), None
    elif pv_mode == "bf16v":
        vp, vs = to_device(v, "bf16"), None          # BF16 V input, never quantized
    elif pv_mode == "mxfp8":                          # V in the token orientation
        vp, vs = lp.lpfa_quantize_mxfp8_varlen(to_device(v, in_dtype), mk, scaling_mode=mode, orientation="tokens")
    else:
        vp, vs = gpu_quantize(lp, v, in_dtype, mk, mode)
    dd = [_descale_tensor(x) for x in descales]
    o, lse = lp.lpfa_attn_fwd_varlen(qp, qs, kp, ks, vp, vs, mq, mk, pv_mode=pv_mode,
                                     q_descale=dd[0], k_descale=dd[1], v_descale=dd[2], workspace=workspace)
    torch.cuda.synchronize()
    return o, lse


def oracle_inputs(q, k, v, lens_q, lens_k, heads, pv_mode="bf16", mode="rceil"):
    """Oracle dequantized Q, K, V (float64) from its own quantizer / cast."""
    pq, sq = omx.quantize_mxfp8_varlen(q, lens_q, mode)
    pk, sk = omx.quantize_mxfp8_varlen(k, lens_k, mode)
    qh = omx.dequantize_mxfp8(pq, sq, lens_q, heads)
    kh = omx.dequantize_mxfp8(pk, sk, lens_k, heads)
    if pv_mode == "fp8":
        vh = omx.e4m3_decode(omx.cast_e4m3(v))
    elif pv_mode == "bf16v":
        vh = np.asarray(v, dtype=np.float64)        # the BF16 values themselves
    elif pv_mode == "mxfp8":
        pv, sv = omx.quantize_mxfp8_varlen_tokens(v, lens_k, mode)
        vh = omx.dequantize_mxfp8_tokens(pv, sv, lens_k, heads)
    else:
        pv, sv = omx.quantize_mxfp8_varlen(v, lens_k, mode)
        vh = omx.dequantize_mxfp8(pv, sv, lens_k, heads)
    return qh, kh, vh


def p_mode_of(pv_mode: str) -> str:
    """The oracle variant that grades a PV mode."""
    return {"fp8": "fp8", "mxfp8": "mxfp8"}.get(pv_mode, "exact")


def oracle_full(q, k, v, lens_q, lens_k, heads, pv_mode="bf16", mode="rceil", descales=(None, None, None)):
    qh, kh, vh = oracle_inputs(q, k, v, lens_q, lens_k, heads, pv_mode, mode)
    qd, kd, vd = [1.0 if x is None else x for x in descales]
    return oatt.attention_fwd(qh, kh, vh, lens_q, lens_k, qd, kd, vd, p_mode=p_mode_of(pv_mode))


def sample_rows(lens_q, heads, seed=0, per_tile_random=2):
    """Seeded (token, head) sample covering every (sequence, head), each 128-row tile's first,
    last and random rows, and every sequence tail."""
    m = ometa.from_lengths(lens_q)
    g = np.random.default_rng(seed)
    toks, hs = [], []
    for i in range(m.num_seqs):
        n = int(m.lengths[i])
        base = int(m.cu_seqlens[i])
        for h in range(heads):
            rows = set()
            for t0 in range(0, n, 128):
                t1 = min(n, t0 + 128) - 1
                rows.update([t0, t1])
                rows.update(g.integers(t0, t1 + 1, size=per_tile_random).tolist())
            rows.add(n - 1)
            for r in sorted(rows):
                toks.append(base + r)
                hs.append(h)
    return np.array(toks), np.array(hs)


def oracle_sampled(q, k, v, lens_q, lens_k, heads, toks, hs, pv_mode="bf16", mode="rceil",
                   descales=(None, None, None)):
    """Oracle O/LSE for sampled query rows (quantizing only what those rows need)."""
    mq = ometa.from_lengths(lens_q)
    mk = ometa.from_lengths(lens_k)
    seq_of_tok = np.searchsorted(mq.cu_seqlens, toks, side="right") - 1
    # query rows
    qp, qe = omx.quantize_rows(q[toks, hs].astype(np.float64), mode)
    qhat = (omx.e4m3_decode(qp).reshape(-1, 4, 32) * np.ldexp(1.0, qe)[..., None]).reshape(-1, 128)
    cache = {}

    def kv(i, h):
        key = (i, h)
        if key not in cache:
            k0, k1 = int(mk.cu_seqlens[i]), int(mk.cu_seqlens[i + 1])
            kp, ke = omx.quantize_rows(k[k0:k1, h].astype(np.float64), mode)
            kh = (omx.e4m3_decode(kp).reshape(-1, 4, 32) * np.ldexp(1.0, ke)[..., None]).reshape(-1, 128)
            if pv_mode == "fp8":
                vh = omx.e4m3_decode(omx.cast_e4m3(v[k0:k1, h]))
            elif pv_mode == "bf16v":
                vh = np.asarray(v[k0:k1, h], dtype=np.float64)
            elif pv_mode == "mxfp8":
                pv, sv = omx.quantize_mxfp8_varlen_tokens(v[k0:k1, h][:, None, :], [k1 - k0], mode)
                vh = omx.dequantize_mxfp8_tokens(pv, sv, [k1 - k0], 1)[:, 0]
            else:
                vp, ve = omx.quantize_rows(v[k0:k1, h].astype(np.float64), mode)
                vh = (omx.e4m3_decode(vp).reshape(-1, 4, 32) * np.ldexp(1.0, ve)[..., None]).reshape(-1, 128)
            cache.clear()
            cache[key] = (kh, vh)
        return cache[key]

    order = np.lexsort((toks, hs, seq_of_tok))
    qd, kd, vd = [1.0 if x is None else x for x in descales]
    o = np.zeros((len(toks), 128))
    l = np.zeros(len(toks))
    oo, ll = oatt.attention_rows(qhat[order], seq_of_tok[order], hs[order],
                                 lambda i, h: kv(i, h)[0], lambda i, h: kv(i, h)[1], lens_k,
                                 qd, kd, vd, p_mode=p_mode_of(pv_mode))
    o[order] = oo
    l[order] = ll
    return o, l


def sampled_backward_reference(q, k, v, o, do, lse, lens_q, lens_k, h, keys, rows, mode="rceil"):
    """Oracle dQ[rows], dK[keys], dV[keys] of head h of a one-sequence problem, from the oracle's
    own MXFP8 quantization of that head (scales are per (token, head, 32 elements), so one head
    quantizes alone) and the definition evaluated row by row. o, do: (T, H, 128); lse: (H, T)."""
    assert len(lens_q) == 1 and len(lens_k) == 1, "one sequence"
    deq = []
    for x, lens in ((q, lens_q), (k, lens_k), (v, lens_k)):
        p, s = omx.quantize_mxfp8_varlen(np.ascontiguousarray(x[:, h:h + 1, :]), lens, mode)
        deq.append(omx.dequantize_mxfp8(p, s, lens, 1)[:, 0, :])
    return obwd.attend_block_backward_sampled(deq[0], deq[1], deq[2], np.asarray(o[:, h], dtype=np.float64),
                                              np.asarray(do[:, h], dtype=np.float64),
                                              np.asarray(lse[h], dtype=np.float64), keys, rows)
