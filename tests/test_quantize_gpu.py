"""Quantizer and cast parity on the GPU: bit-exact against the oracle.

Small ragged cases and adversarial blocks compare the whole payload and the whole padded
scale buffer; the full-size workloads compare every scale pad and a seeded sample of rows.
"""
import numpy as np
import pytest
import torch

import workloads as wl
from oracle import meta as ometa
from oracle import mxfp8 as omx
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import precision_attention_forward_b200 as lp


def _ragged_input(lens, heads, seed, dtype):
    g = np.random.default_rng(seed)
    T = int(np.sum(lens))
    x = g.standard_normal((T, heads, 128)).astype(np.float32)
    x *= (10.0 ** g.uniform(-4, 4, size=(T, heads, 4, 1))).astype(np.float32).repeat(32, axis=3).reshape(T, heads, 128)
    return wl.round_to_bf16(x) if dtype == "bf16" else x


def _check_full(x, lens, heads, dtype, mode):
    meta = lp.lpfa_varlen_meta_from_lengths(lens)
    payload, scales = gu.gpu_quantize(lp, x, dtype, meta, mode)
    ref_p, ref_s = omx.quantize_mxfp8_varlen(x, lens, mode)
    got_p = payload.cpu().numpy()
    got_s = scales.cpu().numpy()
    assert got_s.shape == ref_s.shape
    bad_p = np.argwhere(got_p != ref_p)
    assert bad_p.size == 0, f"{len(bad_p)} payload bytes differ, first at {bad_p[:3].tolist()}"
    bad_s = np.flatnonzero(got_s != ref_s)
    assert bad_s.size == 0, f"{bad_s.size} scale bytes differ, first at {bad_s[:5].tolist()}"


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("mode", ["rceil", "floor"])
def test_quantize_ragged_bit_exact(dtype, mode):
    lens = [1, 127, 128, 129, 300, 64]
    _check_full(_ragged_input(lens, 3, 11, dtype), lens, 3, dtype, mode)


def _adversarial_rows():
    """Rows of 128 values built to hit ties, the 448 boundary, subnormals, signed zeros."""
    vals = omx.e4m3_decode_table()
    finite = np.array([vals[c] for c in range(0x7F)])
    mids = (finite[:-1] + finite[1:]) / 2
    rows = []
    # ties after scaling by 2^-e with e = 0 (amax = 448 in the block)
    blk = np.concatenate([[448.0], mids[:31]])
    rows.append(np.concatenate([blk, -blk, blk[::-1], np.zeros(32)]))
    # amax exactly 448 * 2^e for several e, plus just above
    rows.append(np.concatenate([np.full(32, 448.0 * 2 ** -5), np.full(32, 448.0 * 2 ** 3),
                                np.full(32, np.nextafter(np.float32(448.0), np.float32(1e9)).astype(np.float64)),
                                np.full(32, 1.75)]))
    # subnormal payloads: one large value and many tiny ones in each block
    tiny = np.concatenate([[300.0], np.linspace(-2.0 ** -7, 2.0 ** -7, 31)])
    rows.append(np.concatenate([tiny, tiny * 2 ** 20, tiny * 2 ** -20, -tiny]))
    # signed zeros, negative values that round to zero, an all-zero block, FLOOR saturation
    z = np.zeros(32); z[1::2] = -0.0
    neg_tiny = np.full(32, -1e-4); neg_tiny[0] = 100.0
    sat = np.full(32, 1.9)
    rows.append(np.concatenate([z, neg_tiny, sat, -sat]))
    # huge and tiny magnitudes (fp32 only values get rounded to bf16 for the bf16 case)
    rows.append(np.concatenate([np.full(32, 3.0e38), np.full(32, 1.0e-30), np.full(32, 2.0 ** -133),
                                np.linspace(-1e5, 1e5, 32)]))
    return np.array(rows, dtype=np.float64)


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("mode", ["rceil", "floor"])
def test_quantize_adversarial_bit_exact(dtype, mode):
    rows = _adversarial_rows().astype(np.float32)
    x = np.stack([rows, rows[::-1]], axis=1)  # (5 tokens, 2 heads, 128)
    if dtype == "bf16":
        x = wl.round_to_bf16(x)
    _check_full(x, [5], 2, dtype, mode)
    if dtype == "fp32":  # fp32 subnormal inputs are honoured (no flush to zero)
        sub = np.full((1, 1, 128), np.float32(2.0 ** -140))
        sub[0, 0, ::3] = -np.float32(2.0 ** -147)
        _check_full(sub, [1], 1, dtype, mode)


def test_quantize_strided_input_matches_contiguous():
    lens = [200, 57]
    x = _ragged_input(lens, 4, 5, "bf16")
    meta = lp.lpfa_varlen_meta_from_lengths(lens)
    big = torch.zeros((257, 4, 384), dtype=torch.bfloat16, device="cuda")
    big[:, :, 128:256] = gu.to_device(x, "bf16")
    p1, s1 = lp.lpfa_quantize_mxfp8_varlen(big[:, :, 128:256], meta)
    p2, s2 = lp.lpfa_quantize_mxfp8_varlen(gu.to_device(x, "bf16"), meta)
    assert torch.equal(p1, p2) and torch.equal(s1, s2)
    # head-major storage viewed as (tokens, heads, 128)
    hm = gu.to_device(np.ascontiguousarray(x.transpose(1, 0, 2)), "bf16").transpose(0, 1)
    p3, s3 = lp.lpfa_quantize_mxfp8_varlen(hm, meta)
    assert torch.equal(p3, p2) and torch.equal(s3, s2)


def test_cast_e4m3_bit_exact():
    g = np.random.default_rng(3)
    v = (g.standard_normal((333, 3, 128)) * 10.0 ** g.uniform(-5, 3.5, (333, 3, 1))).astype(np.float32)
    v[0, 0, :4] = [0.0, -0.0, 500.0, -1e4]
    v = wl.round_to_bf16(v)
    out = lp.lpfa_cast_e4m3(gu.to_device(v, "bf16")).cpu().numpy()
    assert np.array_equal(out, omx.cast_e4m3(v))


def _pad_mask(lens, heads):
    m = ometa.from_lengths(lens)
    real = np.zeros(m.total_scale_blocks * heads * 512, dtype=bool)
    for i in range(m.num_seqs):
        n = int(m.lengths[i])
        r = np.arange(n)
        blk = m.scale_off[i] + r // 128
        rr = r % 128
        for h in range(heads):
            base = (blk * heads + h) * 512 + (rr % 32) * 16 + (rr // 32) * 4
            for kb in range(4):
                real[base + kb] = True
    return real


CHUNK_TOKENS = 4096   # a multiple of 128: a chunk's scale atoms are whole atoms of the sequence


def _check_every_byte(x, lens, heads, p_host, s_host, mode, label):
    """Every payload and scale byte of a full-size quantization against the oracle, one 128-aligned
    token chunk of one sequence at a time (the oracle quantizes the chunk as a sequence of its own:
    its blocks are blocks scale_off[i] + t0 / 128 ... of the sequence, with the same atoms, so the
    chunk's scale bytes are one contiguous slice of the storage). Host memory stays bounded."""
    m = ometa.from_lengths(lens)
    assert p_host.shape == x.shape and s_host.size == m.total_scale_blocks * heads * 512
    for i in range(m.num_seqs):
        n, c0 = int(m.lengths[i]), int(m.cu_seqlens[i])
        for t0 in range(0, n, CHUNK_TOKENS):
            t1 = min(n, t0 + CHUNK_TOKENS)
            ref_p, ref_s = omx.quantize_mxfp8_varlen(x[c0 + t0:c0 + t1], [t1 - t0], mode)
            got_p = p_host[c0 + t0:c0 + t1]
            if not np.array_equal(got_p, ref_p):
                bad = np.argwhere(got_p != ref_p)[:3] + [c0 + t0, 0, 0]
                raise AssertionError(f"{label}: payload bytes differ, first at (token, head, channel) {bad.tolist()}")
            b0 = int(m.scale_off[i]) + t0 // 128
            got_s = s_host[b0 * heads * 512:b0 * heads * 512 + ref_s.size]
            if not np.array_equal(got_s, ref_s):
                bad = np.flatnonzero(got_s != ref_s)[:5] + b0 * heads * 512
                raise AssertionError(f"{label}: scale bytes differ, first at byte offsets {bad.tolist()}")


@pytest.mark.parametrize("name", wl.EVAL_ORDER)
def test_quantize_workload(name):
    """Every evaluation workload at full size, in its own dtype and scaling mode: every payload byte
    and every scale byte (pads included) of Q, K and V (LP-FA4 README, "MXFP8 forward and
    backward": E4M3 payload, one E8M0 scale per 32 elements, 128-token-padded scale storage per
    sequence), and every byte of the unscaled E4M3 cast of V in fp8 PV mode."""
    w = wl.WORKLOADS[name]
    lq, lk = wl.lengths(w)
    for which, lens in (("q", lq), ("k", lk), ("v", lk)):
        if which == "v" and w.pv_mode == "fp8":
            continue
        x = wl.make_tensor(w, which)
        dtype = wl.tensor_dtype(w, which)
        meta = lp.lpfa_varlen_meta_from_lengths(lens)
        payload, scales = gu.gpu_quantize(lp, x, dtype, meta, w.scaling_mode)
        p_host, s_host = payload.cpu().numpy(), scales.cpu().numpy()
        del payload, scales
        real = _pad_mask(lens, w.heads)
        assert np.all(s_host[~real] == 0x7F)
        _check_every_byte(x, lens, w.heads, p_host, s_host, w.scaling_mode, f"{name}/{which}")
        del x, p_host, s_host
    if w.pv_mode == "fp8":
        v = wl.make_tensor(w, "v")
        out = lp.lpfa_cast_e4m3(gu.to_device(v, "bf16")).cpu().numpy()
        for t0 in range(0, v.shape[0], CHUNK_TOKENS):
            assert np.array_equal(out[t0:t0 + CHUNK_TOKENS], omx.cast_e4m3(v[t0:t0 + CHUNK_TOKENS])), \
                f"{name}/v cast: bytes differ in tokens [{t0}, {t0 + CHUNK_TOKENS})"


def _check_tokens(x, lens, heads, dtype, mode, xd=None):
    """Token orientation: whole payload and whole scale buffer against the oracle."""
    meta = lp.lpfa_varlen_meta_from_lengths(lens)
    if xd is None:
        xd = gu.to_device(x, dtype)
    payload, scales = lp.lpfa_quantize_mxfp8_varlen(xd, meta, scaling_mode=mode, orientation="tokens")
    ref_p, ref_s = omx.quantize_mxfp8_varlen_tokens(x, lens, mode)
    got_p, got_s = payload.cpu().numpy(), scales.cpu().numpy()
    bad_p = np.argwhere(got_p != ref_p)
    assert bad_p.size == 0, f"{len(bad_p)} payload bytes differ, first at {bad_p[:3].tolist()}"
    bad_s = np.flatnonzero(got_s != ref_s)
    assert bad_s.size == 0, f"{bad_s.size} scale bytes differ, first at {bad_s[:5].tolist()}"
    return payload, scales


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("mode", ["rceil", "floor"])
def test_quantize_tokens_ragged_bit_exact(dtype, mode):
    """Partial and empty 32-token groups, sequences shorter than a group, several blocks."""
    lens = [1, 31, 32, 33, 127, 128, 129, 300, 64]
    _check_tokens(_ragged_input(lens, 3, 12, dtype), lens, 3, dtype, mode)


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("mode", ["rceil", "floor"])
def test_quantize_tokens_adversarial_bit_exact(dtype, mode):
    """The adversarial rows laid along the tokens of each channel (128 tokens, 2 heads)."""
    rows = _adversarial_rows().astype(np.float32)            # (5, 128): values along tokens
    x = np.empty((128, 2, 128), dtype=np.float32)
    for c in range(128):
        x[:, 0, c] = rows[c % 5]
        x[:, 1, c] = rows[(c + 2) % 5][::-1]
    if dtype == "bf16":
        x = wl.round_to_bf16(x)
    _check_tokens(x, [128], 2, dtype, mode)
    _check_tokens(x[:77], [77], 2, dtype, mode)


def test_quantize_tokens_strided_input_matches_contiguous():
    lens = [200, 57]
    x = _ragged_input(lens, 4, 6, "bf16")
    big = torch.zeros((257, 4, 384), dtype=torch.bfloat16, device="cuda")
    big[:, :, 128:256] = gu.to_device(x, "bf16")
    p1, s1 = _check_tokens(x, lens, 4, "bf16", "rceil", xd=big[:, :, 128:256])
    hm = gu.to_device(np.ascontiguousarray(x.transpose(1, 0, 2)), "bf16").transpose(0, 1)
    p2, s2 = _check_tokens(x, lens, 4, "bf16", "rceil", xd=hm)
    assert torch.equal(p1, p2) and torch.equal(s1, s2)


def test_quantize_tokens_workload_v():
    """V of the dense workload (4 x 2048 tokens, 16 heads) at full size, every byte."""
    w = wl.WORKLOADS["dense_4x2048_h16"]
    lq, lk = wl.lengths(w)
    v = wl.make_tensor(w, "v")
    _check_tokens(v, lk, w.heads, "bf16", "rceil")
