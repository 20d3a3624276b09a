"""C-ABI boundary checks that need no GPU: exports, host metadata, argument validation.

Every call here fails validation (or is host-only) before the library touches CUDA.
"""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

import precision_attention_forward_b200 as lp
from oracle import meta as ometa

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "lpfa.h")


def _declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"LPFA_API\s+[\w\s\*]+?\b(lpfa_\w+)\s*\(", text)))


def test_every_declared_symbol_is_exported():
    names = _declared_functions()
    assert len(names) == len(lp.EXPORTED_SYMBOLS)
    assert set(names) == set(lp.EXPORTED_SYMBOLS)
    lib = ctypes.CDLL(lp.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n


def test_version_and_sizes():
    assert "sm_100a" in lp.lpfa_version()
    assert lp._lib.lpfa_meta_dev_ints(5) == 12
    assert lp._lib.lpfa_meta_dev_ints(0) == 0


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_fill_host_matches_oracle(seed):
    g = np.random.default_rng(seed)
    lens = g.integers(1, 5000, size=g.integers(1, 40))
    m = lp.lpfa_varlen_meta_fill_host(lens)
    o = ometa.from_lengths(lens)
    assert m.cu_seqlens.tolist() == o.cu_seqlens.tolist()
    assert m.scale_off.tolist() == o.scale_off.tolist()
    assert (m.num_seqs, m.total_tokens, m.total_scale_blocks, m.max_seqlen) == (
        o.num_seqs, o.total_tokens, o.total_scale_blocks, o.max_seqlen)
    assert m.scale_bytes(7) == o.total_scale_blocks * 7 * 512


@pytest.mark.parametrize("lens", [[], [0], [5, -1], [3, 0, 4]])
def test_fill_host_rejects_bad_lengths(lens):
    with pytest.raises(lp.LpfaError) as ei:
        lp.lpfa_varlen_meta_fill_host(lens)
    assert ei.value.status == lp.LPFA_ERR_INVALID_ARG


def test_fill_host_rejects_overflow():
    with pytest.raises(lp.LpfaError):
        lp.lpfa_varlen_meta_fill_host([2 ** 31 - 1, 5])


def _fake_meta(n, tokens):
    m = lp._Meta()
    m.num_seqs, m.total_tokens, m.total_scale_blocks, m.max_seqlen = n, tokens, (tokens + 127) // 128, tokens
    m.dev = 0x1000  # never dereferenced: validation fails first
    return m


FAKE = 0x10000  # an aligned, never-dereferenced "device" address


def _attn(**over):
    args = dict(q=FAKE, q_sf=FAKE, k=FAKE, k_sf=FAKE, v=FAKE, v_sf=FAKE, mq=_fake_meta(2, 300), mk=_fake_meta(2, 300),
                heads=4, head_dim=128, pv=0, qd=None, kd=None, vd=None, out=FAKE, lse=FAKE)
    args.update(over)
    st = lp._lib.lpfa_attn_fwd_varlen(args["q"], args["q_sf"], args["k"], args["k_sf"], args["v"], args["v_sf"],
                                      ctypes.byref(args["mq"]), ctypes.byref(args["mk"]), args["heads"],
                                      args["head_dim"], args["pv"], args["qd"], args["kd"], args["vd"],
                                      args["out"], args["lse"], None)
    return st, lp._lib.lpfa_last_error_message().decode()


@pytest.mark.parametrize("over,needle", [
    (dict(head_dim=64), "head_dim"),
    (dict(heads=0), "heads"),
    (dict(pv=7), "pv_mode"),
    (dict(pv=1), "v_sf"),                 # fp8 PV mode with V scale factors
    (dict(v_sf=None), "v_sf"),            # bf16 PV mode without them
    (dict(mk=_fake_meta(3, 300)), "sequences"),
    (dict(q=None), "NULL"),
    (dict(lse=FAKE + 4), "aligned"),
])
def test_attention_argument_validation(over, needle):
    st, msg = _attn(**over)
    assert st == lp.LPFA_ERR_INVALID_ARG
    assert needle in msg


def test_quantize_argument_validation():
    m = _fake_meta(1, 100)
    f = lp._lib.lpfa_quantize_mxfp8_varlen
    assert f(FAKE, 0, 2048, 128, 16, 64, ctypes.byref(m), 0, FAKE, FAKE, None) == lp.LPFA_ERR_INVALID_ARG
    assert f(FAKE, 5, 2048, 128, 16, 128, ctypes.byref(m), 0, FAKE, FAKE, None) == lp.LPFA_ERR_INVALID_ARG
    assert f(FAKE, 0, 2048, 128, 16, 128, ctypes.byref(m), 9, FAKE, FAKE, None) == lp.LPFA_ERR_INVALID_ARG
    assert f(FAKE, 0, 2047, 128, 16, 128, ctypes.byref(m), 0, FAKE, FAKE, None) == lp.LPFA_ERR_INVALID_ARG
    assert f(None, 0, 2048, 128, 16, 128, ctypes.byref(m), 0, FAKE, FAKE, None) == lp.LPFA_ERR_INVALID_ARG
    empty = lp._Meta()
    assert f(FAKE, 0, 2048, 128, 16, 128, ctypes.byref(empty), 0, FAKE, FAKE, None) == lp.LPFA_ERR_INVALID_ARG


def test_cast_argument_validation():
    f = lp._lib.lpfa_cast_e4m3
    assert f(FAKE, 2048, 128, 10, 16, 100, FAKE, None) == lp.LPFA_ERR_INVALID_ARG
    assert f(FAKE, 2048, 128, 0, 16, 128, FAKE, None) == lp.LPFA_ERR_INVALID_ARG
    assert f(FAKE + 2, 2048, 128, 10, 16, 128, FAKE, None) == lp.LPFA_ERR_INVALID_ARG


def test_descaled_entry_rejects_negative_strides():
    good = lp._Descale(FAKE, 0, 1)
    bad = lp._Descale(FAKE, -1, 0)
    for descs in ((bad, None, None), (None, None, bad)):
        ptrs = [ctypes.byref(d) if d is not None else None for d in descs]
        st = lp._lib.lpfa_attn_fwd_varlen_descaled(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                                   ctypes.byref(_fake_meta(2, 300)), ctypes.byref(_fake_meta(2, 300)),
                                                   4, 128, 0, *ptrs, FAKE, FAKE, None)
        assert st == lp.LPFA_ERR_INVALID_ARG
        assert "stride" in lp._lib.lpfa_last_error_message().decode()
    # a valid descriptor passes descale validation and fails later (head_dim), not on the strides
    st = lp._lib.lpfa_attn_fwd_varlen_descaled(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                               ctypes.byref(_fake_meta(2, 300)), ctypes.byref(_fake_meta(2, 300)),
                                               4, 64, 0, ctypes.byref(good), None, None, FAKE, FAKE, None)
    assert st == lp.LPFA_ERR_INVALID_ARG and "head_dim" in lp._lib.lpfa_last_error_message().decode()


@pytest.mark.parametrize("shape,want", [
    ((1,), (0, 0)), ((), (0, 0)), ((1, 1), (0, 0)), ((4,), (0, 1)), ((1, 4), (0, 1)),
    ((3, 4), (4, 1)), ((3, 1), (1, 0)),
])
def test_descale_strides_shapes(shape, want):
    t = torch.ones(shape, dtype=torch.float32)
    assert lp.descale_strides(t, 3, 4) == want


def test_descale_strides_views_and_rejects():
    base = torch.arange(12, dtype=torch.float32).reshape(4, 3)
    assert lp.descale_strides(base.t(), 3, 4) == (1, 3)            # transposed (S, H) view
    assert lp.descale_strides(torch.ones(1).expand(3, 4), 3, 4) == (0, 0)
    assert lp.descale_strides(torch.ones(4).expand(3, 4), 3, 4) == (0, 1)
    for bad in (torch.ones(5), torch.ones(2, 4), torch.ones(3, 4, dtype=torch.float64), torch.ones(3, 4, 1)):
        with pytest.raises(ValueError):
            lp.descale_strides(bad, 3, 4)


def _bwd(**over):
    args = dict(q=FAKE, q_sf=FAKE, k=FAKE, k_sf=FAKE, v=FAKE, v_sf=FAKE, out=FAKE, dout=FAKE, lse=FAKE,
                mq=_fake_meta(2, 300), mk=_fake_meta(2, 300), heads=4, head_dim=128, qd=None, kd=None, vd=None,
                dq=FAKE, dk=FAKE, dv=FAKE, dk_sf=None, dv_sf=None, mx=0)
    args.update(over)
    st = lp._lib.lpfa_attn_bwd_varlen(args["q"], args["q_sf"], args["k"], args["k_sf"], args["v"], args["v_sf"],
                                      args["out"], args["dout"], args["lse"], ctypes.byref(args["mq"]),
                                      ctypes.byref(args["mk"]), args["heads"], args["head_dim"], args["qd"],
                                      args["kd"], args["vd"], args["dq"], args["dk"], args["dv"], args["dk_sf"],
                                      args["dv_sf"], args["mx"], None)
    return st, lp._lib.lpfa_last_error_message().decode()


@pytest.mark.parametrize("over,needle", [
    (dict(q=None), "NULL"),
    (dict(v_sf=None), "NULL"),
    (dict(dq=None), "NULL"),
    (dict(mx=2), "output_mxfp8_dkv"),
    (dict(mx=1), "dk_sf"),                      # MXFP8 dK/dV without their scale buffers
    (dict(head_dim=64), "head_dim"),
    (dict(heads=0), "heads"),
    (dict(mk=_fake_meta(3, 300)), "sequences"),
    (dict(dq=FAKE + 8), "aligned"),
    (dict(qd=ctypes.pointer(lp._Descale(FAKE, -1, 0))), "stride"),
])
def test_backward_argument_validation(over, needle):
    st, msg = _bwd(**over)
    assert st == lp.LPFA_ERR_INVALID_ARG
    assert needle in msg


def test_shared_query_rejects_several_query_sequences():
    """lpfa_attn_fwd_shared_q takes a query metadata of exactly one sequence (checked before any
    CUDA call)."""
    host_q = np.zeros(2 * 3, dtype=np.int32)
    host_k = np.zeros(2 * 3, dtype=np.int32)
    cq, ck = lp._Meta(), lp._Meta()
    lens = np.array([5, 7], dtype=np.int32)
    assert lp._lib.lpfa_varlen_meta_fill_host(lens.ctypes.data, 2, host_q.ctypes.data, ctypes.byref(cq)) == 0
    assert lp._lib.lpfa_varlen_meta_fill_host(lens.ctypes.data, 2, host_k.ctypes.data, ctypes.byref(ck)) == 0
    cq.dev = ck.dev = 16   # never dereferenced: validation fails first
    one = lp._Descale(None, 0, 0)
    st = lp._lib.lpfa_attn_fwd_shared_q(16, 16, 16, 16, 16, 16, ctypes.byref(cq), ctypes.byref(ck), 1, 128, 0,
                                        ctypes.byref(one), ctypes.byref(one), ctypes.byref(one), 16, 16, None)
    assert st == lp.LPFA_ERR_INVALID_ARG
    assert b"one sequence" in lp._lib.lpfa_last_error_message()


def _attn_ws(ws, ws_bytes, pv=0):
    one = lp._Descale(None, 0, 0)
    mq, mk = _fake_meta(2, 300), _fake_meta(2, 300)
    st = lp._lib.lpfa_attn_fwd_varlen_ws(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE if pv == 0 else None, ctypes.byref(mq),
                                         ctypes.byref(mk), 4, 128, pv, ctypes.byref(one), ctypes.byref(one),
                                         ctypes.byref(one), FAKE, FAKE, ws, ctypes.c_size_t(ws_bytes), None)
    return st, lp._lib.lpfa_last_error_message().decode()


def test_workspace_size_and_validation():
    """bf16 PV mode over a workspace needs total_tokens(K) * heads * 256 bytes, 16-byte aligned;
    the other modes need none (checked before any CUDA call)."""
    mk = _fake_meta(2, 300)
    assert lp._lib.lpfa_attn_fwd_workspace_bytes(ctypes.byref(mk), 4, 0) == 300 * 4 * 256
    for pv in (1, 2, 3):
        assert lp._lib.lpfa_attn_fwd_workspace_bytes(ctypes.byref(mk), 4, pv) == 0
    assert lp._lib.lpfa_attn_fwd_workspace_bytes(None, 4, 0) == 0
    need = 300 * 4 * 256
    for ws, nbytes, needle in ((None, need, "workspace"), (FAKE + 8, need, "aligned"),
                               (FAKE, need - 1, "too small")):
        st, msg = _attn_ws(ws, nbytes)
        assert st == lp.LPFA_ERR_INVALID_ARG and needle in msg, msg


def test_dequantize_argument_validation():
    m = _fake_meta(1, 10)
    for args, needle in (((None, FAKE, 2, 128, FAKE), "NULL"), ((FAKE, FAKE, 2, 64, FAKE), "head_dim"),
                         ((FAKE, FAKE, 0, 128, FAKE), "heads"), ((FAKE, FAKE, 2, 128, FAKE + 2), "aligned")):
        st = lp._lib.lpfa_dequantize_mxfp8_varlen(args[0], args[1], ctypes.byref(m), args[2], args[3], args[4], None)
        assert st == lp.LPFA_ERR_INVALID_ARG and needle in lp._lib.lpfa_last_error_message().decode()


def test_shared_query_workspace_validation():
    """lpfa_attn_fwd_shared_q_ws checks its bf16-PV workspace like the varlen entry point."""
    host_q = np.zeros(2 * 2, dtype=np.int32)
    host_k = np.zeros(2 * 3, dtype=np.int32)
    cq, ck = lp._Meta(), lp._Meta()
    assert lp._lib.lpfa_varlen_meta_fill_host(np.array([300], np.int32).ctypes.data, 1, host_q.ctypes.data,
                                              ctypes.byref(cq)) == 0
    assert lp._lib.lpfa_varlen_meta_fill_host(np.array([5, 7], np.int32).ctypes.data, 2, host_k.ctypes.data,
                                              ctypes.byref(ck)) == 0
    cq.dev = ck.dev = 16
    one = lp._Descale(None, 0, 0)
    st = lp._lib.lpfa_attn_fwd_shared_q_ws(16, 16, 16, 16, 16, 16, ctypes.byref(cq), ctypes.byref(ck), 2, 128, 0,
                                           ctypes.byref(one), ctypes.byref(one), ctypes.byref(one), 16, 16, None,
                                           ctypes.c_size_t(0), None)
    assert st == lp.LPFA_ERR_INVALID_ARG
    assert b"workspace" in lp._lib.lpfa_last_error_message()


def test_noalloc_size_limit_is_checked_before_device_work():
    """Beyond the scratch size, bf16 PV is rejected with the sizes before any device work (the
    pointers here are never dereferenced)."""
    H, tokens = 16, (64 << 20) // (256 * 16) + 1
    ck = _fake_meta(1, tokens)
    cq = _fake_meta(1, 128)
    one = lp._Descale(None, 0, 0)
    st = lp._lib.lpfa_attn_fwd_varlen_noalloc(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ctypes.byref(cq), ctypes.byref(ck),
                                              H, 128, 0, ctypes.byref(one), ctypes.byref(one), ctypes.byref(one),
                                              FAKE, FAKE, None)
    assert st == lp.LPFA_ERR_INVALID_ARG
    assert b"scratch" in lp._lib.lpfa_last_error_message()


def test_binding_workspace_choice():
    """The binding's workspace argument: False/None mean in-kernel V conversion, other modes need
    none, and a given tensor must be a large enough contiguous uint8 buffer (checked on the host)."""
    meta = lp.lpfa_varlen_meta_fill_host([300, 5])
    need = lp.lpfa_attn_fwd_workspace_bytes(meta, 4, "bf16")
    assert need == 305 * 4 * 256
    assert lp.lpfa_attn_fwd_workspace_bytes(meta, 4, "fp8") == 0
    assert lp._workspace(False, meta, 4, "bf16", "cpu") is None
    assert lp._workspace(None, meta, 4, "bf16", "cpu") is None
    assert lp._workspace(True, meta, 4, "fp8", "cpu") is None
    ok = torch.empty(need, dtype=torch.uint8)
    assert lp._workspace(ok, meta, 4, "bf16", "cpu") is ok
    for bad in (torch.empty(need - 1, dtype=torch.uint8), torch.empty(need, dtype=torch.int8),
                torch.empty(2 * need, dtype=torch.uint8)[::2]):
        with pytest.raises(ValueError):
            lp._workspace(bad, meta, 4, "bf16", "cpu")
