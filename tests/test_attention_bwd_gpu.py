"""Attention backward on the GPU against the oracle (oracle/backward.py).

The forward runs first (bf16 PV mode, MXFP8 V in the head_dim orientation); its O and LSE, the
seeded dO and the oracle's own dequantization of the same inputs feed the oracle backward, so
the comparison isolates the backward. Gradients have no unit scale, so the bounds are relative:
rel-L2 <= 1e-2 and max-abs <= 2e-2 of the reference's largest magnitude (P and dS enter the
MMAs as BF16), with an absolute floor of 1e-4 for gradients that vanish by construction.
"""
import numpy as np
import pytest
import torch

import workloads as wl
from oracle import backward as obwd
from oracle import mxfp8 as omx
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import precision_attention_forward_b200 as lp

REL_L2 = 1e-2
REL_MAX = 2e-2


def _grad_close(got, ref, label):
    """Relative bounds with an absolute floor of 1e-4 in the denominators: a gradient that is
    zero by construction (one key: every softmax row is constant, dQ = dK = 0) is judged by its
    absolute rounding residue."""
    got = np.asarray(got, dtype=np.float64)
    floor = 1e-4
    scale = max(float(np.max(np.abs(ref))), floor)
    rel = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), floor * np.sqrt(max(ref.size, 1))))
    mx = float(np.max(np.abs(got - ref))) / scale if got.size else 0.0
    assert rel <= REL_L2 and mx <= REL_MAX, f"{label}: rel-L2 {rel:.3e}, max-abs/max {mx:.3e}"
    return rel, mx


def _run(lq, lk, H, seed, descales=(None, None, None), mx_dkv=False):
    q, k, v = wl.small_random(seed, lq, lk, H)
    g = np.random.default_rng(seed + 1000)
    do = wl.round_to_bf16(g.standard_normal((sum(lq), H, 128)).astype(np.float32))
    mq = lp.lpfa_varlen_meta_from_lengths(lq)
    mk = lp.lpfa_varlen_meta_from_lengths(lk)
    qp, qs = gu.gpu_quantize(lp, q, "bf16", mq)
    kp, ks = gu.gpu_quantize(lp, k, "bf16", mk)
    vp, vs = gu.gpu_quantize(lp, v, "bf16", mk)
    dd = [gu._descale_tensor(x) for x in descales]
    o, lse = lp.lpfa_attn_fwd_varlen(qp, qs, kp, ks, vp, vs, mq, mk, pv_mode="bf16",
                                     q_descale=dd[0], k_descale=dd[1], v_descale=dd[2])
    res = lp.lpfa_attn_bwd_varlen(qp, qs, kp, ks, vp, vs, o, gu.to_device(do, "bf16"), lse, mq, mk,
                                  q_descale=dd[0], k_descale=dd[1], v_descale=dd[2], output_mxfp8_dkv=mx_dkv)
    torch.cuda.synchronize()
    assert lp.lpfa_device_status() == (lp.LPFA_OK, 0)
    qh, kh, vh = gu.oracle_inputs(q, k, v, lq, lk, H)
    qd, kd, vd = [1.0 if x is None else x for x in descales]
    ref = obwd.attention_bwd(qh, kh, vh, o.float().cpu().numpy().astype(np.float64), do.astype(np.float64),
                             lse.cpu().numpy().astype(np.float64), lq, lk, qd, kd, vd)
    return res, ref


CASES = [
    ([1], [1], 1),
    ([5], [5], 2),
    ([128], [128], 2),
    ([129], [200], 1),
    ([300, 77, 1], [300, 77, 1], 2),
    ([200], [1000], 2),
    ([64, 700], [513, 129], 2),
]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_backward_small_cases(case):
    lq, lk, H = CASES[case]
    (dq, dk, dv), (rq, rk, rv) = _run(lq, lk, H, 300 + case)
    for name, got, ref in (("dQ", dq, rq), ("dK", dk, rk), ("dV", dv, rv)):
        _grad_close(got.float().cpu().numpy(), ref, f"{name} {lq}/{lk}")


@pytest.mark.parametrize("descales", [(0.5, 3.0, 0.25), (-1.0, 1.0, 2.0),
                                      (np.array([0.5, -1.25]), np.array([[1.0, 0.75], [2.0, 1.0]]), np.array([1.0, 2.0]))])
def test_backward_descales(descales):
    lq, lk, H = [300, 77], [129, 200], 2
    (dq, dk, dv), (rq, rk, rv) = _run(lq, lk, H, 350, descales=descales)
    for name, got, ref in (("dQ", dq, rq), ("dK", dk, rk), ("dV", dv, rv)):
        _grad_close(got.float().cpu().numpy(), ref, f"{name} descales")


def test_backward_mxfp8_dkv_output():
    """output_mxfp8_dkv: dK and dV as E4M3 + E8M0 (head_dim orientation); dequantized, within the
    gradient bound plus E4M3 rounding of the block maximum."""
    lq, lk, H = [300, 77], [129, 200], 2
    (dq, dk, dv, dk_sf, dv_sf), (rq, rk, rv) = _run(lq, lk, H, 360, mx_dkv=True)
    _grad_close(dq.float().cpu().numpy(), rq, "dQ")
    for name, pl, sc, ref in (("dK", dk, dk_sf, rk), ("dV", dv, dv_sf, rv)):
        deq = omx.dequantize_mxfp8(pl.cpu().numpy(), sc.cpu().numpy(), lk, H)
        rel = float(np.linalg.norm(deq - ref) / np.linalg.norm(ref))
        assert rel <= 5e-2, f"{name} MXFP8: rel-L2 {rel:.3e}"
        # every block within E4M3 rounding (2^-4 of its maximum) plus the gradient bound
        bmax = np.abs(ref).reshape(-1, 4, 32).max(axis=2, keepdims=True)
        err = np.abs(deq - ref).reshape(-1, 4, 32)
        assert np.all(err <= bmax * 2.0 ** -4 + REL_MAX * np.max(np.abs(ref))), name


def test_backward_repeated_runs_bit_identical():
    lq, lk, H = [300, 77], [129, 200], 2
    (a, _) = _run(lq, lk, H, 370)
    (b, _) = _run(lq, lk, H, 370)
    for x, y in zip(a, b):
        assert torch.equal(x.view(torch.int16), y.view(torch.int16))


def test_backward_dense_workload():
    """The dense workload (4 x 2048, 16 heads) at full size."""
    w = wl.WORKLOADS["dense_4x2048_h16"]
    lq, lk = wl.lengths(w)
    q, k, v = (wl.make_tensor(w, x) for x in "qkv")
    g = np.random.default_rng(9)
    do = wl.round_to_bf16(g.standard_normal(q.shape).astype(np.float32))
    mq = lp.lpfa_varlen_meta_from_lengths(lq)
    mk = lp.lpfa_varlen_meta_from_lengths(lk)
    qp, qs = gu.gpu_quantize(lp, q, "bf16", mq)
    kp, ks = gu.gpu_quantize(lp, k, "bf16", mk)
    vp, vs = gu.gpu_quantize(lp, v, "bf16", mk)
    o, lse = lp.lpfa_attn_fwd_varlen(qp, qs, kp, ks, vp, vs, mq, mk, pv_mode="bf16")
    dq, dk, dv = lp.lpfa_attn_bwd_varlen(qp, qs, kp, ks, vp, vs, o, gu.to_device(do, "bf16"), lse, mq, mk)
    torch.cuda.synchronize()
    assert lp.lpfa_device_status() == (lp.LPFA_OK, 0)
    qh, kh, vh = gu.oracle_inputs(q, k, v, lq, lk, w.heads)
    rq, rk, rv = obwd.attention_bwd(qh, kh, vh, o.float().cpu().numpy().astype(np.float64), do.astype(np.float64),
                                    lse.cpu().numpy().astype(np.float64), lq, lk)
    for name, got, ref in (("dQ", dq, rq), ("dK", dk, rk), ("dV", dv, rv)):
        print(name, _grad_close(got.float().cpu().numpy(), ref, f"{name} dense"))

