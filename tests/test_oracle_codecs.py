"""Pins for the oracle's E4M3 / E8M0 codecs and MXFP8 quantizer (CPU only).

Each check compares the oracle with something other than itself: hand-picked
values from the 8-bit float definition, brute-force nearest search over all 256
codes, brute-force exponent search, and torch's own float8_e4m3fn conversion (an
independent library implementation of the same format).
"""
import math

import numpy as np
import pytest
import torch

from oracle import meta as ometa
from oracle import mxfp8 as omx
from tests.conftest import read_golden


def _finite_table():
    vals = omx.e4m3_decode_table()
    codes = [c for c in range(256) if not math.isnan(vals[c])]
    return vals, codes


def test_decode_matches_torch_float8():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = omx.e4m3_decode_table()
    both_nan = np.isnan(ref) & np.isnan(ours)
    assert np.all(both_nan | (ref == ours))
    assert np.isnan(ours[0x7F]) and np.isnan(ours[0xFF])
    assert int(np.isnan(ours).sum()) == 2


def test_decode_structure():
    vals, _ = _finite_table()
    pos = vals[:0x7F]
    assert np.all(np.diff(pos) > 0), "positive codes must be strictly increasing"
    for c in range(0x7F):
        assert vals[c | 0x80] == -vals[c] or (c == 0 and math.copysign(1, vals[0x80]) < 0)
    assert vals[0x7E] == 448.0 and vals[0x01] == 2.0 ** -9 and vals[0x08] == 2.0 ** -6


def _brute_encode(x):
    """Nearest finite E4M3 value, ties to the even code, saturating; sign kept."""
    vals, codes = _finite_table()
    a = abs(x)
    if a >= 448.0:
        best = 0x7E
    else:
        best, bestd = None, None
        for c in range(0x7F):
            d = abs(vals[c] - a)
            if bestd is None or d < bestd or (d == bestd and c % 2 == 0):
                best, bestd = c, d
    return best | (0x80 if math.copysign(1.0, x) < 0 else 0)


def test_encode_handpicked(golden):
    for value, code, *_ in read_golden("e4m3_handpicked.txt"):
        got = int(omx.e4m3_encode(np.array([float(value)]))[0])
        assert got == int(code, 16), (value, hex(got), code)
        assert _brute_encode(float(value)) == int(code, 16), value


def test_encode_brute_force_grid():
    vals, _ = _finite_table()
    finite = np.array([vals[c] for c in range(0x7F)])
    mids = (finite[:-1] + finite[1:]) / 2            # every tie point
    probes = np.concatenate([finite, mids, np.nextafter(mids, 0), np.nextafter(mids, 1e9),
                             [448.0, 460.0, 464.0, 470.0, 500.0, 1e6, 2.0 ** -12, 1e-30]])
    probes = np.concatenate([probes, -probes])
    got = omx.e4m3_encode(probes)
    for x, g in zip(probes, got):
        assert int(g) == _brute_encode(float(x)), (x, hex(int(g)))


def test_encode_matches_torch_in_range():
    g = np.random.default_rng(1)
    x = np.concatenate([g.standard_normal(20000) * s for s in (1e-3, 0.1, 1, 30, 200)])
    x = x.astype(np.float32)
    x = x[np.abs(x) < 464.0]                          # torch's cast gives NaN beyond, no satfinite
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = omx.e4m3_encode(x.astype(np.float64))
    assert np.array_equal(ref, ours)


def _brute_rceil(amax):
    if amax == 0:
        return -127
    for e in range(-127, 128):
        if amax <= 448.0 * 2.0 ** e:
            return e
    raise AssertionError


def _brute_floor(amax):
    if amax == 0:
        return -127
    e = 0
    while 2.0 ** e > amax:
        e -= 1
    while 2.0 ** (e + 1) <= amax:
        e += 1
    return max(-127, min(127, e - 8))


def test_e8m0_handpicked(golden):
    for amax, mode, e, byte, code, *_ in read_golden("e8m0_handpicked.txt"):
        got = int(omx.e8m0_exponent(np.array([float(amax)]), mode)[0])
        assert got == int(e) and got + 127 == int(byte), (amax, mode, got)
        payload = omx.e4m3_encode(np.array([float(amax) * 2.0 ** -got]))[0]
        assert int(payload) == int(code, 16), (amax, mode, hex(int(payload)))


def test_e8m0_brute_force():
    g = np.random.default_rng(2)
    am = np.concatenate([
        np.abs(g.standard_normal(3000)) * 10.0 ** g.uniform(-40, 38, 3000),
        448.0 * 2.0 ** np.arange(-130, 120, dtype=np.float64),
        np.nextafter(448.0 * 2.0 ** np.arange(-100, 100, dtype=np.float64), 1e300),
        2.0 ** np.arange(-149, 128, dtype=np.float64),
        [0.0, 2.0 ** -149, 3.4e38],
    ]).astype(np.float32).astype(np.float64)
    r = omx.e8m0_exponent(am, "rceil")
    f = omx.e8m0_exponent(am, "floor")
    for a, er, ef in zip(am, r, f):
        assert int(er) == max(-127, _brute_rceil(float(a))), a
        assert int(ef) == _brute_floor(float(a)), a


def test_quantize_matches_torch_division_path():
    """RCEIL payload equals torch's float8 cast of x / 2^e (no saturation is reachable)."""
    g = np.random.default_rng(3)
    x = (g.standard_normal((300, 3, 128)) * 10.0 ** g.uniform(-3, 3, (300, 3, 1))).astype(np.float32)
    lens = [1, 130, 169]
    payload, scales = omx.quantize_mxfp8_varlen(x, lens, "rceil")
    e = omx.scale_exponents(scales, lens, 3)
    blocks = torch.from_numpy(x.reshape(300, 3, 4, 32).astype(np.float64))
    ref = (blocks / torch.from_numpy(2.0 ** e.astype(np.float64))[..., None]).to(torch.float32)
    ref = ref.to(torch.float8_e4m3fn).view(torch.uint8).reshape(300, 3, 128).numpy()
    assert np.array_equal(ref, payload)
    # minimality: with e - 1 the block maximum would not fit
    amax = np.abs(x.reshape(300, 3, 4, 32)).max(axis=3).astype(np.float64)
    assert np.all(amax <= 448.0 * 2.0 ** e)
    assert np.all(amax > 448.0 * 2.0 ** (e - 1))


def test_quantize_power_of_two_invariance():
    g = np.random.default_rng(4)
    x = g.standard_normal((200, 2, 128)).astype(np.float32)
    lens = [77, 123]
    for mode in ("rceil", "floor"):
        p0, s0 = omx.quantize_mxfp8_varlen(x, lens, mode)
        p1, s1 = omx.quantize_mxfp8_varlen(x * np.float32(8.0), lens, mode)
        assert np.array_equal(p0, p1)
        e0 = omx.scale_exponents(s0, lens, 2)
        e1 = omx.scale_exponents(s1, lens, 2)
        assert np.array_equal(e1, e0 + 3)


def test_quantize_floor_saturates():
    row = np.zeros((1, 1, 128), dtype=np.float32)
    row[0, 0, :32] = 1.9            # FLOOR: 1.9 * 256 > 448 -> 448
    row[0, 0, 32:64] = -1.9
    p, s = omx.quantize_mxfp8_varlen(row, [1], "floor")
    assert set(p[0, 0, :32].tolist()) == {0x7E}
    assert set(p[0, 0, 32:64].tolist()) == {0xFE}
    assert set(p[0, 0, 64:].tolist()) == {0x00}
    e = omx.scale_exponents(s, [1], 1)
    assert e[0, 0].tolist() == [-8, -8, -127, -127]


def test_scale_storage_layout_by_hand():
    """Place three distinct exponents by hand and find them at the documented byte offsets."""
    lens = [3, 130]                 # sequence 1 spans two 128-token blocks
    H = 2
    x = np.zeros((133, H, 128), dtype=np.float32)
    # sequence 0, token 2, head 1, block kb=3 -> amax 448 * 2^5 -> e = 5
    x[2, 1, 96] = 448.0 * 32
    # sequence 1, token 129 (block 1, row 1), head 0, kb=0 -> amax 448 * 2^-3 -> e = -3
    x[3 + 129, 0, 0] = 448.0 / 8
    # sequence 1, token 40 (block 0, row 40), head 1, kb=2 -> amax 448 -> e = 0
    x[3 + 40, 1, 64] = 448.0
    payload, scales = omx.quantize_mxfp8_varlen(x, lens, "rceil")
    m = ometa.from_lengths(lens)
    assert m.total_scale_blocks == 3 and scales.size == 3 * H * 512
    # seq 0 uses block 0; seq 1 uses blocks 1 and 2
    off_a = ((0 * H + 1) * 512) + (2 % 32) * 16 + (2 // 32) * 4 + 3
    off_b = ((2 * H + 0) * 512) + (1 % 32) * 16 + (1 // 32) * 4 + 0
    off_c = ((1 * H + 1) * 512) + (40 % 32) * 16 + (40 // 32) * 4 + 2
    assert scales[off_a] == 127 + 5
    assert scales[off_b] == 127 - 3
    assert scales[off_c] == 127
    # every other real row holds 0 (all-zero blocks), pads hold 0x7F
    real = np.zeros_like(scales, dtype=bool)
    for i, n in enumerate(lens):
        for r in range(n):
            b, rr = m.scale_off[i] + r // 128, r % 128
            for h in range(H):
                for kb in range(4):
                    real[((b * H + h) * 512) + (rr % 32) * 16 + (rr // 32) * 4 + kb] = True
    assert real.sum() == 133 * H * 4
    assert np.all(scales[~real] == 0x7F)
    special = {off_a, off_b, off_c}
    for o in np.flatnonzero(real):
        if int(o) not in special:
            assert scales[o] == 0
    assert payload[2, 1, 96] == 0x7E and payload[3 + 129, 0, 0] == 0x7E


def test_dequantize_round_trip_error():
    g = np.random.default_rng(5)
    x = g.standard_normal((256, 2, 128)).astype(np.float32)
    p, s = omx.quantize_mxfp8_varlen(x, [256], "rceil")
    xh = omx.dequantize_mxfp8(p, s, [256], 2)
    e = omx.scale_exponents(s, [256], 2)
    # half an E4M3 ulp (relative 2^-4) for normals, plus the subnormal floor 2^-10 * 2^e
    bound = np.maximum(np.abs(x).reshape(256, 2, 4, 32) * 2.0 ** -4,
                       2.0 ** (e - 10)[..., None]).reshape(256, 2, 128)
    assert np.all(np.abs(xh - x) <= bound)


def test_cast_e4m3_matches_torch():
    g = np.random.default_rng(6)
    v = (g.standard_normal(50000) * 2).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(omx.cast_e4m3(v), ref)


def test_negative_tiny_keeps_sign():
    x = np.array([-1e-6, -0.0, 1e-6, -2.0 ** -11])
    assert omx.e4m3_encode(x).tolist() == [0x80, 0x80, 0x00, 0x80]


def test_token_orientation_is_head_dim_orientation_of_the_transpose():
    """Token-orientation quantization of a 128-token block equals the head_dim-orientation row
    quantization of its transpose (channels as rows, tokens as the 128 elements), for every
    32-token group that holds tokens; partial last blocks pad the transpose with zeros, which
    leaves the group maxima alone."""
    g = np.random.default_rng(40)
    lens, H = [300, 37, 128], 2
    x = (g.standard_normal((sum(lens), H, 128)) * np.exp2(g.integers(-6, 7, size=(1, H, 128)))).astype(np.float32)
    p, s = omx.quantize_mxfp8_varlen_tokens(x, lens)
    m = ometa.from_lengths(lens)
    for i in range(m.num_seqs):
        c0, n = int(m.cu_seqlens[i]), int(m.lengths[i])
        for b in range(0, n, 128):
            nb = min(128, n - b)
            for h in range(H):
                blk = np.zeros((128, 128))
                blk[:, :nb] = x[c0 + b:c0 + b + nb, h].astype(np.float64).T   # (channel, token)
                rp, re = omx.quantize_rows(blk)
                assert np.array_equal(p[c0 + b:c0 + b + nb, h], rp[:, :nb].T)
                base = ((m.scale_off[i] + b // 128) * H + h) * 512
                for grp in range(4):
                    for c in range(128):
                        byte = s[base + (c % 32) * 16 + (c // 32) * 4 + grp]
                        if grp * 32 < nb:
                            assert byte == re[c, grp] + 127
                        else:
                            assert byte == 0x7F          # group with no token of the sequence


def test_token_orientation_layout_by_hand():
    """One channel with a known per-token magnitude: its group scales sit at the stated bytes."""
    lens, H = [70], 1
    x = np.zeros((70, 1, 128), dtype=np.float32)
    x[:, 0, 5] = np.arange(1, 71, dtype=np.float32)            # channel 5: token t holds t + 1
    x[:, 0, 100] = -3.0                                          # channel 100: constant
    p, s = omx.quantize_mxfp8_varlen_tokens(x, lens)
    # channel 5: group maxima 32, 64, 70 -> RCEIL e = -3, -2, -2 (448 * 2^-3 = 56 >= 32 ...)
    for grp, want in ((0, omx.e8m0_exponent(32.0)), (1, omx.e8m0_exponent(64.0)), (2, omx.e8m0_exponent(70.0))):
        assert s[(5 % 32) * 16 + (5 // 32) * 4 + grp] == int(want) + 127
    assert s[(5 % 32) * 16 + (5 // 32) * 4 + 3] == 0x7F          # tokens 96..127 do not exist
    assert s[(100 % 32) * 16 + (100 // 32) * 4 + 0] == int(omx.e8m0_exponent(3.0)) + 127
    assert s[(0 % 32) * 16 + 0] == 0x00                          # an all-zero channel: amax 0
    xh = omx.dequantize_mxfp8_tokens(p, s, lens, H)
    assert np.array_equal(xh[:, 0, 100], np.full(70, -3.0))
    assert np.array_equal(xh[:, 0, 5], np.arange(1, 71, dtype=np.float64) * 0 + xh[:, 0, 5])
    assert np.all(np.abs(xh[:, 0, 5] - np.arange(1, 71)) <= np.arange(1, 71) / 16)
