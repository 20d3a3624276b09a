"""Pins of the attention backward oracle (oracle/backward.py): finite differences of the
forward oracle, closed forms, and structural identities."""
import math

import numpy as np
import pytest

from oracle import attention as oatt
from oracle import backward as obwd
from oracle import mxfp8 as omx


def _loss(q, k, v, do, qd, kd, vd):
    o, _ = oatt.attend_block(q, k, v, qd, kd, vd)
    return float(np.sum(o * do))


@pytest.mark.parametrize("descales", [(1.0, 1.0, 1.0), (0.7, -1.3, 2.0)])
def test_gradients_match_central_differences(descales):
    """L = sum(O * dO) of the forward definition: its numerical gradient with respect to
    sampled coordinates of q, k and v equals the backward's dQ, dK, dV."""
    qd, kd, vd = descales
    g = np.random.default_rng(50)
    q, k, v = g.standard_normal((3, 128)), g.standard_normal((5, 128)), g.standard_normal((5, 128))
    do = g.standard_normal((3, 128))
    o, lse = oatt.attend_block(q, k, v, qd, kd, vd)
    dq, dk, dv = obwd.attend_block_backward(q, k, v, o, do, lse, qd, kd, vd)
    eps = 1e-6
    for name, x, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for _ in range(12):
            idx = (int(g.integers(x.shape[0])), int(g.integers(128)))
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args = {"q": q, "k": k, "v": v}
            lp_ = _loss(*(xp if n == name else args[n] for n in "qkv"), do, qd, kd, vd)
            lm_ = _loss(*(xm if n == name else args[n] for n in "qkv"), do, qd, kd, vd)
            num = (lp_ - lm_) / (2 * eps)
            assert abs(num - grad[idx]) <= 1e-6 * max(1.0, abs(num)), (name, idx, num, grad[idx])


def test_single_key_closed_form():
    """One key: p = 1 for every row, so dQ = dK = 0 and dV = vd * sum of dO."""
    g = np.random.default_rng(51)
    q, k, v, do = g.standard_normal((4, 128)), g.standard_normal((1, 128)), g.standard_normal((1, 128)), g.standard_normal((4, 128))
    o, lse = oatt.attend_block(q, k, v, vd=1.5)
    dq, dk, dv = obwd.attend_block_backward(q, k, v, o, do, lse, vd=1.5)
    assert np.allclose(dq, 0.0, atol=1e-12) and np.allclose(dk, 0.0, atol=1e-12)
    assert np.allclose(dv[0], 1.5 * do.sum(axis=0), atol=1e-12)


def test_key_shift_invariance_and_d_identity():
    """With the forward's exact O, D_r = sum_j p_rj dP_rj, so each row of dS sums to zero and dQ
    does not change when every key is shifted by the same vector (the logits of a row move by a
    constant, p does not change)."""
    g = np.random.default_rng(52)
    q, k, v, do = (g.standard_normal((6, 128)), g.standard_normal((40, 128)), g.standard_normal((40, 128)),
                   g.standard_normal((6, 128)))
    o, lse = oatt.attend_block(q, k, v)
    dq, dk, dv = obwd.attend_block_backward(q, k, v, o, do, lse)
    shift = g.standard_normal(128)
    o2, lse2 = oatt.attend_block(q, k + shift, v)
    dq2, _, _ = obwd.attend_block_backward(q, k + shift, v, o2, do, lse2)
    assert np.allclose(dq, dq2, atol=1e-9)
    # D_r = sum_j p dP
    s = (q @ k.T) / math.sqrt(128)
    p = np.exp(s - lse[:, None])
    assert np.allclose(np.sum(do * o, axis=1), np.sum(p * (do @ v.T), axis=1), atol=1e-12)


def test_packing_matches_separate_sequences():
    g = np.random.default_rng(53)
    lq, lk, H = [5, 3], [7, 2], 2
    q = g.standard_normal((8, H, 128)); k = g.standard_normal((9, H, 128)); v = g.standard_normal((9, H, 128))
    do = g.standard_normal((8, H, 128))
    o, lse = oatt.attention_fwd(q, k, v, lq, lk)
    dq, dk, dv = obwd.attention_bwd(q, k, v, o, do, lse, lq, lk)
    a = obwd.attend_block_backward(q[5:, 1], k[7:, 1], v[7:, 1], o[5:, 1], do[5:, 1], lse[1, 5:])
    assert np.allclose(dq[5:, 1], a[0]) and np.allclose(dk[7:, 1], a[1]) and np.allclose(dv[7:, 1], a[2])


def test_mxfp8_dkv_output_round_trip():
    """output_mxfp8_dkv: dK, dV as head_dim-orientation MXFP8, within E4M3 precision of the
    block maximum."""
    g = np.random.default_rng(54)
    lens = [70, 33]
    dk = g.standard_normal((103, 2, 128)) * 1e-3
    dv = g.standard_normal((103, 2, 128))
    (pk, sk), (pv, sv) = obwd.quantize_dkv(dk, dv, lens)
    for x, pl, sc in ((dk, pk, sk), (dv, pv, sv)):
        xh = omx.dequantize_mxfp8(pl, sc, lens, 2)
        bmax = np.abs(x).reshape(103, 2, 4, 32).max(axis=3, keepdims=True)
        err = np.abs(xh - x).reshape(103, 2, 4, 32)
        assert np.all(err <= bmax * 2.0 ** -4 + 1e-300)
