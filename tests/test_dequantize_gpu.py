"""MXFP8 -> BF16 dequantization on the GPU, and the bf16 PV mode over a workspace.

lpfa_dequantize_mxfp8_varlen gives E4M3(payload) * 2^(byte - 127) (LP-FA4 README, "MXFP8 forward
and backward": the payload times its block's E8M0 power of two), rounded once to BF16. The
oracle's float64 dequantization (oracle/mxfp8.py: dequantize_mxfp8) is exact; its value is
representable in FP32 (4 significant bits, exponent >= -136) or overflows it, so rounding it
through FP32 to BF16 must give the kernel's bits exactly, every code and scale byte included.

The bf16 PV mode computes the same thing two ways: V dequantized once into a caller workspace
(lpfa_attn_fwd_varlen_ws, the default of the binding) or each V tile converted inside the
attention kernel (lpfa_attn_fwd_varlen_descaled). The two must agree bit for bit; the oracle
grades the result at the forward's tolerances (the other attention tests use the workspace path).
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


def _random_mx(seed, lengths, heads, scale_lo=0, scale_hi=254):
    """Random E4M3 codes (no NaN code) and scale bytes over the padded storage of `lengths`."""
    rng = np.random.default_rng(seed)
    m = ometa.from_lengths(lengths)
    T = int(m.total_tokens)
    codes = rng.integers(0, 256, size=(T, heads, 128), dtype=np.uint8)
    codes[(codes & 0x7F) == 0x7F] ^= 0x01          # 0x7F / 0xFF (NaN) -> 0x7E / 0xFE
    scales = rng.integers(scale_lo, scale_hi + 1, size=int(m.total_scale_blocks) * heads * 512, dtype=np.uint8)
    return codes, scales


def _bits(x: torch.Tensor) -> np.ndarray:
    return x.contiguous().view(torch.int16).cpu().numpy()


@pytest.mark.parametrize("lengths,heads,lo,hi", [
    ([1], 1, 0, 254),
    ([5, 128, 129], 2, 0, 254),               # every scale byte: subnormal results, overflow to inf
    ([300, 1, 77, 256, 513], 3, 100, 150),    # ordinary magnitudes, ragged tails
    ([2048] * 3, 4, 0, 254),
])
def test_dequantize_matches_oracle_bitwise(lengths, heads, lo, hi):
    codes, scales = _random_mx(7 + len(lengths), lengths, heads, lo, hi)
    meta = lp.lpfa_varlen_meta_from_lengths(lengths)
    out = lp.lpfa_dequantize_mxfp8_varlen(torch.from_numpy(codes).cuda(), torch.from_numpy(scales).cuda(), meta)
    torch.cuda.synchronize()
    ref = omx.dequantize_mxfp8(codes, scales, lengths, heads)           # exact, float64
    ref_bf16 = torch.from_numpy(ref).to(torch.float32).to(torch.bfloat16)
    got, want = _bits(out), _bits(ref_bf16)
    bad = np.argwhere(got != want)
    assert bad.size == 0, "%d mismatches, first at %s: got 0x%04x want 0x%04x (value %r)" % (
        len(bad), tuple(bad[0]), got[tuple(bad[0])] & 0xFFFF, want[tuple(bad[0])] & 0xFFFF, ref[tuple(bad[0])])


def test_dequantize_of_the_quantizer_is_exact():
    """Quantize then dequantize: the BF16 result is the oracle's exact x_hat (no rounding at all)."""
    lengths, heads = [700, 129, 1], 4
    x = np.random.default_rng(3).standard_normal((sum(lengths), heads, 128)).astype(np.float32) * 3
    xb = torch.from_numpy(x).to(torch.bfloat16)
    x = xb.float().numpy()
    meta = lp.lpfa_varlen_meta_from_lengths(lengths)
    payload, scales = lp.lpfa_quantize_mxfp8_varlen(xb.cuda(), meta)
    out = lp.lpfa_dequantize_mxfp8_varlen(payload, scales, meta)
    torch.cuda.synchronize()
    pq, sq = omx.quantize_mxfp8_varlen(x, lengths)
    ref = omx.dequantize_mxfp8(pq, sq, lengths, heads)
    np.testing.assert_array_equal(out.double().cpu().numpy(), ref)


CASES = [
    ([1], [1], 1),
    ([129], [129], 1),
    ([300, 77, 1], [300, 77, 1], 3),
    ([200], [1000], 2),
    ([64, 700], [513, 129], 2),
    ([256] * 9, [384] * 9, 2),
]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_bf16_workspace_path_matches_in_kernel_conversion(case):
    lq, lk, H = CASES[case]
    q, k, v = wl.small_random(1000 + case, lq, lk, H)
    o_ws, l_ws = gu.run_path(lp, q, k, v, lq, lk, H, pv_mode="bf16")
    o_in, l_in = gu.run_path(lp, q, k, v, lq, lk, H, pv_mode="bf16", workspace=False)
    assert torch.equal(o_ws.view(torch.int16), o_in.view(torch.int16))
    assert torch.equal(l_ws.view(torch.int32), l_in.view(torch.int32))
    o_ref, l_ref = gu.oracle_full(q, k, v, lq, lk, H, pv_mode="bf16")
    gu.assert_within(gu.compare_attention(o_in, l_in, o_ref, l_ref), f"in-kernel V conversion {lq}/{lk}")
    assert lp.lpfa_device_status() == (lp.LPFA_OK, 0)


def test_bf16_workspace_path_with_descales_and_shared_query():
    lq, lk, H = [300], [300], 2
    q, k, v = wl.small_random(77, lq, lk, H)
    d = (np.array([0.5, 2.0], np.float32), None, np.array([[1.5, -0.25]], np.float32))
    o_ws, l_ws = gu.run_path(lp, q, k, v, lq, lk, H, pv_mode="bf16", descales=d)
    o_in, l_in = gu.run_path(lp, q, k, v, lq, lk, H, pv_mode="bf16", descales=d, workspace=False)
    assert torch.equal(o_ws.view(torch.int16), o_in.view(torch.int16))
    assert torch.equal(l_ws.view(torch.int32), l_in.view(torch.int32))

    Lq, lks = 200, [129, 700, 1]
    q, k, v = wl.small_random(78, [Lq], lks, H)
    mq = lp.lpfa_varlen_meta_from_lengths([Lq])
    mk = lp.lpfa_varlen_meta_from_lengths(lks)
    qp, qs = gu.gpu_quantize(lp, q, "bf16", mq)
    kp, ks = gu.gpu_quantize(lp, k, "bf16", mk)
    vp, vs = gu.gpu_quantize(lp, v, "bf16", mk)
    outs = [lp.lpfa_attn_fwd_shared_q(qp, qs, kp, ks, vp, vs, mq, mk, pv_mode="bf16", workspace=w) for w in (True, False)]
    torch.cuda.synchronize()
    assert torch.equal(outs[0][0].view(torch.int16), outs[1][0].view(torch.int16))
    assert torch.equal(outs[0][1].view(torch.int32), outs[1][1].view(torch.int32))
    assert lp.lpfa_device_status() == (lp.LPFA_OK, 0)


def test_workspace_is_checked_and_reusable():
    lq, lk, H = [300, 5], [260, 9], 2
    q, k, v = wl.small_random(5, lq, lk, H)
    mq = lp.lpfa_varlen_meta_from_lengths(lq)
    mk = lp.lpfa_varlen_meta_from_lengths(lk)
    qp, qs = gu.gpu_quantize(lp, q, "bf16", mq)
    kp, ks = gu.gpu_quantize(lp, k, "bf16", mk)
    vp, vs = gu.gpu_quantize(lp, v, "bf16", mk)
    need = lp.lpfa_attn_fwd_workspace_bytes(mk, H, "bf16")
    assert need == sum(lk) * H * 256
    with pytest.raises(ValueError):
        lp.lpfa_attn_fwd_varlen(qp, qs, kp, ks, vp, vs, mq, mk, pv_mode="bf16",
                                workspace=torch.empty(need - 16, dtype=torch.uint8, device="cuda"))
    # The same workspace (garbage-filled first) serves two calls; each call rewrites what it reads.
    ws = torch.full((need + 4096,), 0xFF, dtype=torch.uint8, device="cuda")
    o1, l1 = lp.lpfa_attn_fwd_varlen(qp, qs, kp, ks, vp, vs, mq, mk, pv_mode="bf16", workspace=ws)
    o2, l2 = lp.lpfa_attn_fwd_varlen(qp, qs, kp, ks, vp, vs, mq, mk, pv_mode="bf16", workspace=ws)
    o3, l3 = lp.lpfa_attn_fwd_varlen(qp, qs, kp, ks, vp, vs, mq, mk, pv_mode="bf16", workspace=False)
    torch.cuda.synchronize()
    for o, l in ((o1, l1), (o2, l2)):
        assert torch.equal(o.view(torch.int16), o3.view(torch.int16))
        assert torch.equal(l.view(torch.int32), l3.view(torch.int32))
    assert lp.lpfa_device_status() == (lp.LPFA_OK, 0)


def test_dequantize_writes_only_its_output():
    """The BF16 output sits inside a pattern-filled buffer; every guard byte must survive, and rows
    of every sequence (ragged tails included) must be written."""
    lengths, heads = [129, 1, 300], 3
    codes, scales = _random_mx(21, lengths, heads, 100, 150)
    meta = lp.lpfa_varlen_meta_from_lengths(lengths)
    T = sum(lengths)
    n = T * heads * 128 * 2
    guard = 4096
    buf = torch.full((n + 2 * guard,), 0xA5, dtype=torch.uint8, device="cuda")
    out = buf[guard:guard + n].view(torch.bfloat16).view(T, heads, 128)
    lp.lpfa_dequantize_mxfp8_varlen(torch.from_numpy(codes).cuda(), torch.from_numpy(scales).cuda(), meta, out=out)
    torch.cuda.synchronize()
    host = buf.cpu().numpy()
    assert (host[:guard] == 0xA5).all() and (host[guard + n:] == 0xA5).all()
    ref = torch.from_numpy(omx.dequantize_mxfp8(codes, scales, lengths, heads)).to(torch.float32).to(torch.bfloat16)
    assert torch.equal(out.cpu().view(torch.int16), ref.view(torch.int16))
