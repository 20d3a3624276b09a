"""The forward entry point that allocates nothing (lpfa_attn_fwd_varlen_noalloc).

It exists for callers that cannot give the library device memory: code inside a host runtime
whose own memory pool owns the GPU and forbids other allocations, and latency-critical paths where
a cudaMalloc / cudaFree (which can synchronise the device) is not allowed. In bf16 PV mode it puts
the BF16 copy of V into a fixed scratch array inside the library instead of a caller workspace.

The GPU test calls it through the C ABI twice in a row, on two different problems (the second
smaller than the first, so stale scratch from the first call would show), and compares each
result with the ordinary entry point's (lpfa_attn_fwd_varlen_descaled, V converted inside the
attention kernel) at the forward's tolerances and bit for bit. This file is collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads as wl
from tests import gpu_util as gu

if torch.cuda.is_available():
    import precision_attention_forward_b200 as lp
else:  # the size check below needs no GPU
    lp = pytest.importorskip("precision_attention_forward_b200")

SCRATCH_BYTES = 64 << 20


def _inputs(seed, lq, lk, H, pv_mode):
    q, k, v = wl.small_random(seed, lq, lk, H)
    mq = lp.lpfa_varlen_meta_from_lengths(lq)
    mk = lp.lpfa_varlen_meta_from_lengths(lk)
    qp, qs = gu.gpu_quantize(lp, q, "bf16", mq)
    kp, ks = gu.gpu_quantize(lp, k, "bf16", mk)
    if pv_mode == "fp8":
        vp, vs = lp.lpfa_cast_e4m3(gu.to_device(v, "bf16")), None
    else:
        vp, vs = gu.gpu_quantize(lp, v, "bf16", mk)
    return (qp, qs, kp, ks, vp, vs, mq, mk)


def _noalloc(ins, H, pv_mode):
    qp, qs, kp, ks, vp, vs, mq, mk = ins
    T = mq.total_tokens
    out = torch.empty((T, H, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((H, T), dtype=torch.float32, device="cuda")
    one = lp._Descale(None, 0, 0)
    st = lp._lib.lpfa_attn_fwd_varlen_noalloc(
        qp.data_ptr(), qs.data_ptr(), kp.data_ptr(), ks.data_ptr(), vp.data_ptr(),
        vs.data_ptr() if vs is not None else None, ctypes.byref(mq._c), ctypes.byref(mk._c), H, 128,
        lp.PV_MODES[pv_mode], ctypes.byref(one), ctypes.byref(one), ctypes.byref(one), out.data_ptr(),
        lse.data_ptr(), None)
    assert st == lp.LPFA_OK, lp._lib.lpfa_last_error_message().decode()
    return out, lse


def _existing(ins, pv_mode):
    qp, qs, kp, ks, vp, vs, mq, mk = ins
    return lp.lpfa_attn_fwd_varlen(qp, qs, kp, ks, vp, vs, mq, mk, pv_mode=pv_mode, workspace=False)


@pytest.mark.gpu
def test_noalloc_matches_existing_entry_point_on_two_calls_in_a_row():
    cases = [(11, [700, 129, 1], [900, 300, 5], 3, "bf16"),   # ragged, cross, several KV tiles
             (12, [256, 40], [130, 64], 2, "bf16")]           # smaller: reuses the first call's scratch
    for seed, lq, lk, H, pv_mode in cases:
        ins = _inputs(seed, lq, lk, H, pv_mode)
        o, l = _noalloc(ins, H, pv_mode)
        o_ref, l_ref = _existing(ins, pv_mode)
        torch.cuda.synchronize()
        gu.assert_within(gu.compare_attention(o, l, o_ref.double().cpu().numpy(), l_ref.double().cpu().numpy()),
                         f"no-allocation entry point {lq}/{lk}")
        assert torch.equal(o.view(torch.int16), o_ref.view(torch.int16))
        assert torch.equal(l.view(torch.int32), l_ref.view(torch.int32))
    assert lp.lpfa_device_status() == (lp.LPFA_OK, 0)


@pytest.mark.gpu
def test_noalloc_modes_without_scratch():
    ins = _inputs(13, [300], [500], 2, "fp8")
    o, l = _noalloc(ins, 2, "fp8")
    o_ref, l_ref = _existing(ins, "fp8")
    torch.cuda.synchronize()
    assert torch.equal(o.view(torch.int16), o_ref.view(torch.int16))
    assert torch.equal(l.view(torch.int32), l_ref.view(torch.int32))


def test_noalloc_rejects_problems_beyond_its_scratch():
    """Key tokens x heads x 256 bytes above the fixed scratch: a clear error before any work (no GPU
    call is made, so this runs on the CPU too)."""
    H = 16
    tokens = SCRATCH_BYTES // (256 * H) + 1
    ck = lp._Meta()
    ck.num_seqs, ck.total_tokens, ck.total_scale_blocks, ck.max_seqlen = 1, tokens, (tokens + 127) // 128, tokens
    ck.dev = 16
    cq = lp._Meta()
    cq.num_seqs, cq.total_tokens, cq.total_scale_blocks, cq.max_seqlen, cq.dev = 1, 128, 1, 128, 16
    one = lp._Descale(None, 0, 0)
    st = lp._lib.lpfa_attn_fwd_varlen_noalloc(16, 16, 16, 16, 16, 16, ctypes.byref(cq), ctypes.byref(ck), H, 128,
                                              lp.PV_MODES["bf16"], ctypes.byref(one), ctypes.byref(one),
                                              ctypes.byref(one), 16, 16, None)
    assert st == lp.LPFA_ERR_INVALID_ARG
    msg = lp._lib.lpfa_last_error_message().decode()
    assert "scratch" in msg and str(SCRATCH_BYTES) in msg
