"""C-ABI boundary checks that need no GPU: exports, host metadata, argument validation.

Every call here fails validation (or is host-only) before the library touches CUDA.
"""
import ctypes
import os
import re

import numpy as np
import pytest

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
