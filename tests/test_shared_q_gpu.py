"""Shared-query forward on the GPU (lpfa_attn_fwd_shared_q).

Reading of the LP-FA4 README's "shared-query workloads" (opening paragraph; not defined there):
one query sequence is shared by n key/value sequences, and block i of the output is the attention
of the query set over key/value sequence i. Graded against the oracle
(oracle/attention.py: attention_fwd_shared_q) at the forward's tolerances, and bit for bit
against the ordinary varlen call with the query sequence repeated once per key/value sequence.
"""
import numpy as np
import pytest
import torch

import workloads as wl
from oracle import attention as oatt
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import precision_attention_forward_b200 as lp


def _v_device(lp, v, pv_mode, mk):
    if pv_mode == "fp8":
        return lp.lpfa_cast_e4m3(gu.to_device(v, "bf16")), None
    if pv_mode == "bf16v":
        return gu.to_device(v, "bf16"), None
    if pv_mode == "mxfp8":
        return lp.lpfa_quantize_mxfp8_varlen(gu.to_device(v, "bf16"), mk, orientation="tokens")
    return gu.gpu_quantize(lp, v, "bf16", mk)


def _shared(q, k, v, Lq, lk, pv_mode, descales=(None, None, None)):
    mq = lp.lpfa_varlen_meta_from_lengths([Lq])
    mk = lp.lpfa_varlen_meta_from_lengths(lk)
    qp, qs = gu.gpu_quantize(lp, q, "bf16", mq)
    kp, ks = gu.gpu_quantize(lp, k, "bf16", mk)
    vp, vs = _v_device(lp, v, pv_mode, mk)
    dd = [gu._descale_tensor(x) for x in descales]
    o, lse = lp.lpfa_attn_fwd_shared_q(qp, qs, kp, ks, vp, vs, mq, mk, pv_mode=pv_mode,
                                       q_descale=dd[0], k_descale=dd[1], v_descale=dd[2])
    torch.cuda.synchronize()
    assert lp.lpfa_device_status() == (lp.LPFA_OK, 0)
    return o, lse


CASES = [
    (300, [129, 700, 1, 256, 513], 2),   # a query pair and a single tile; ragged and one-key sequences
    (128, [1000], 1),
    (1, [5, 3], 3),
    (257, [300] * 5, 2),
]


@pytest.mark.parametrize("pv_mode", ["bf16", "fp8", "bf16v", "mxfp8"])
@pytest.mark.parametrize("case", range(len(CASES)))
def test_shared_query_matches_oracle(pv_mode, case):
    Lq, lk, H = CASES[case]
    q, _, _ = wl.small_random(400 + case, [Lq], [1], H)
    _, k, v = wl.small_random(500 + case, [1], lk, H)
    if pv_mode == "fp8":
        v = v * np.float32(2.0)
    o, lse = _shared(q, k, v, Lq, lk, pv_mode)
    qh, kh, vh = gu.oracle_inputs(q, k, v, [Lq], lk, H, pv_mode)
    o_ref, lse_ref = oatt.attention_fwd_shared_q(qh, kh, vh, lk, p_mode=gu.p_mode_of(pv_mode))
    gu.assert_within(gu.compare_attention(o, lse, o_ref, lse_ref), f"shared q {pv_mode} {Lq}/{lk}")


@pytest.mark.parametrize("pv_mode", ["bf16", "fp8"])
def test_shared_query_per_sequence_descales(pv_mode):
    """Descales indexed by (key/value sequence, head)."""
    Lq, lk, H = 200, [129, 400, 77], 2
    q, _, _ = wl.small_random(41, [Lq], [1], H)
    _, k, v = wl.small_random(42, [1], lk, H)
    if pv_mode == "fp8":
        v = v * np.float32(2.0)
    qd = np.array([0.5, -1.25])
    kd = np.array([[1.0, 0.75], [2.0, 1.0], [0.25, 1.5]])
    vd = np.array([[1.0, -2.0]])
    o, lse = _shared(q, k, v, Lq, lk, pv_mode, descales=(qd, kd, vd))
    qh, kh, vh = gu.oracle_inputs(q, k, v, [Lq], lk, H, pv_mode)
    o_ref, lse_ref = oatt.attention_fwd_shared_q(qh, kh, vh, lk, qd, kd, vd, p_mode=gu.p_mode_of(pv_mode))
    gu.assert_within(gu.compare_attention(o, lse, o_ref, lse_ref, o_scale=np.abs(vd).reshape(1, H, 1)),
                     f"shared q descales {pv_mode}")


@pytest.mark.parametrize("pv_mode", ["bf16", "fp8", "mxfp8"])
def test_shared_query_equals_repeated_queries_bitwise(pv_mode):
    """The shared query set gives the same bits as the varlen call on the query sequence repeated
    once per key/value sequence (the per-tile arithmetic does not depend on the schedule)."""
    Lq, lk, H = 300, [129, 700, 1, 256], 2
    q, _, _ = wl.small_random(61, [Lq], [1], H)
    _, k, v = wl.small_random(62, [1], lk, H)
    if pv_mode == "fp8":
        v = v * np.float32(2.0)
    o, lse = _shared(q, k, v, Lq, lk, pv_mode)
    qrep = np.concatenate([q] * len(lk))
    o2, lse2 = gu.run_path(lp, qrep, k, v, [Lq] * len(lk), lk, H, pv_mode=pv_mode)
    assert torch.equal(o.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(lse.view(torch.int32), lse2.view(torch.int32))


def test_shared_query_many_sequences():
    """More key/value sequences than the longest-first order holds (plain order)."""
    g = np.random.default_rng(7)
    lk = g.integers(1, 200, size=300).tolist()
    Lq, H = 130, 1
    q, _, _ = wl.small_random(71, [Lq], [1], H)
    _, k, v = wl.small_random(72, [1], lk, H)
    o, lse = _shared(q, k, v, Lq, lk, "bf16")
    qh, kh, vh = gu.oracle_inputs(q, k, v, [Lq], lk, H, "bf16")
    o_ref, lse_ref = oatt.attention_fwd_shared_q(qh, kh, vh, lk)
    gu.assert_within(gu.compare_attention(o, lse, o_ref, lse_ref), "shared q, 300 sequences")


def test_shared_query_outputs_stay_inside_their_buffers():
    """O (n*Lq, H, 128) and LSE (H, n*Lq) inside pattern-filled guard bytes."""
    from tests.test_failure_gpu import _guarded, _guards_intact
    Lq, lk, H = 300, [129, 700, 1], 2
    q, _, _ = wl.small_random(81, [Lq], [1], H)
    _, k, v = wl.small_random(82, [1], lk, H)
    mq = lp.lpfa_varlen_meta_from_lengths([Lq])
    mk = lp.lpfa_varlen_meta_from_lengths(lk)
    qp, qs = gu.gpu_quantize(lp, q, "bf16", mq)
    kp, ks = gu.gpu_quantize(lp, k, "bf16", mk)
    vp, vs = gu.gpu_quantize(lp, v, "bf16", mk)
    rows = Lq * len(lk)
    ob, ov = _guarded(rows * H * 128 * 2)
    lb, lv = _guarded(H * rows * 4)
    out = ov.view(torch.bfloat16).view(rows, H, 128)
    lse = lv.view(torch.float32).view(H, rows)
    lp.lpfa_attn_fwd_shared_q(qp, qs, kp, ks, vp, vs, mq, mk, out=out, lse=lse)
    torch.cuda.synchronize()
    assert lp.lpfa_device_status() == (lp.LPFA_OK, 0)
    assert _guards_intact(ob, ov.numel()) and _guards_intact(lb, lv.numel())
    qh, kh, vh = gu.oracle_inputs(q, k, v, [Lq], lk, H)
    o_ref, lse_ref = oatt.attention_fwd_shared_q(qh, kh, vh, lk)
    gu.assert_within(gu.compare_attention(out, lse, o_ref, lse_ref), "guarded shared q")
