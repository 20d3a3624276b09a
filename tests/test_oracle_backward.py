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


def test_sampled_rows_match_full_backward_and_finite_differences():
    """attend_block_backward_sampled: its rows equal the full backward's on a case with descales,
    and its dK/dQ rows match central differences of the forward definition."""
    g = np.random.default_rng(71)
    q, k, v = g.standard_normal((37, 128)), g.standard_normal((29, 128)), g.standard_normal((29, 128))
    do = g.standard_normal((37, 128))
    qd, kd, vd = 0.8, 1.1, -0.6
    o, lse = oatt.attend_block(q, k, v, qd, kd, vd)
    keys, rows = [0, 5, 28], [0, 17, 36]
    sq, sk, sv = obwd.attend_block_backward_sampled(q, k, v, o, do, lse, keys, rows, qd, kd, vd)
    fq, fk, fv = obwd.attend_block_backward(q, k, v, o, do, lse, qd, kd, vd)
    np.testing.assert_allclose(sq, fq[rows], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(sk, fk[keys], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(sv, fv[keys], rtol=1e-12, atol=1e-12)
    eps = 1e-6
    for name, x, grad, idx_rows in (("q", q, sq, rows), ("k", k, sk, keys), ("v", v, sv, keys)):
        for t, row in enumerate(idx_rows):
            col = int(g.integers(128))
            xp, xm = x.copy(), x.copy()
            xp[row, col] += eps
            xm[row, col] -= eps
            args = {"q": q, "k": k, "v": v}
            lp_ = _loss(*(xp if n == name else args[n] for n in "qkv"), do, qd, kd, vd)
            lm_ = _loss(*(xm if n == name else args[n] for n in "qkv"), do, qd, kd, vd)
            num = (lp_ - lm_) / (2 * eps)
            assert abs(num - grad[t, col]) <= 1e-6 * max(1.0, abs(num)), (name, row, col, num, grad[t, col])


def test_sampled_reference_helper_matches_full_oracle():
    """tests.gpu_util.sampled_backward_reference (used at the video shape on the GPU): per-head
    quantization and sampled rows equal the full varlen oracle's rows on a small two-head case."""
    from tests import gpu_util as gu
    import workloads as wl

    lq, lk, H = [300], [260], 2
    q, k, v = wl.small_random(5, lq, lk, H)
    qh, kh, vh = gu.oracle_inputs(q, k, v, lq, lk, H)
    o_full, lse = oatt.attention_fwd(qh, kh, vh, lq, lk)
    g = np.random.default_rng(6)
    o = o_full.astype(np.float32)
    do = g.standard_normal(q.shape).astype(np.float32)
    fq, fk, fv = obwd.attention_bwd(qh, kh, vh, o.astype(np.float64), do.astype(np.float64), lse, lq, lk)
    keys, rows = [0, 127, 128, 259], [0, 1, 255, 299]
    for h in range(H):
        sq, sk, sv = gu.sampled_backward_reference(q, k, v, o, do, lse, lq, lk, h, keys, rows)
        np.testing.assert_allclose(sq, fq[rows, h], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(sk, fk[keys, h], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(sv, fv[keys, h], rtol=1e-10, atol=1e-12)
