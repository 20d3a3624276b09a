"""Pins for the oracle's attention forward and metadata (CPU only).

Closed forms, a brute-force pure-Python softmax, scipy's logsumexp and
invariances tie the oracle to the mathematics rather than to itself.
"""
import math

import numpy as np
import pytest
from scipy.special import logsumexp

from oracle import attention as oatt
from oracle import meta as ometa
from oracle import mxfp8 as omx

SCALE = 1.0 / math.sqrt(128.0)


def test_meta_prefix_sums_by_hand():
    m = ometa.from_lengths([5, 128, 129, 300])
    assert m.cu_seqlens.tolist() == [0, 5, 133, 262, 562]
    assert m.scale_off.tolist() == [0, 1, 2, 4, 7]
    assert (m.num_seqs, m.total_tokens, m.total_scale_blocks, m.max_seqlen) == (4, 562, 7, 300)
    with pytest.raises(ValueError):
        ometa.from_lengths([3, 0])
    with pytest.raises(ValueError):
        ometa.from_lengths([])


def test_constant_v_gives_v():
    g = np.random.default_rng(0)
    q, k = g.standard_normal((7, 128)), g.standard_normal((33, 128))
    vrow = g.standard_normal(128)
    v = np.tile(vrow, (33, 1))
    o, _ = oatt.attend_block(q, k, v)
    assert np.allclose(o, vrow[None, :], atol=1e-12, rtol=0)


def test_single_key():
    g = np.random.default_rng(1)
    q, k, v = g.standard_normal((5, 128)), g.standard_normal((1, 128)), g.standard_normal((1, 128))
    o, lse = oatt.attend_block(q, k, v, qd=0.5, kd=3.0)
    assert np.allclose(o, v, atol=1e-12, rtol=0)
    s = (q @ k[0]) * 0.5 * 3.0 * SCALE
    assert np.allclose(lse, s, atol=1e-12, rtol=0)


def test_equal_logits():
    g = np.random.default_rng(2)
    n = 57
    q = g.standard_normal((4, 128))
    k = np.tile(g.standard_normal(128), (n, 1))
    v = g.standard_normal((n, 128))
    o, lse = oatt.attend_block(q, k, v)
    s = (q @ k[0]) * SCALE
    assert np.allclose(lse, np.log(n) + s, atol=1e-12, rtol=0)
    assert np.allclose(o, v.mean(axis=0)[None, :], atol=1e-12, rtol=0)


def _brute_attention(q, k, v, qd=1.0, kd=1.0, vd=1.0):
    """Pure-Python loops: softmax(q.k * scale) v, natural-log LSE."""
    out, lse = [], []
    for r in range(len(q)):
        s = []
        for j in range(len(k)):
            acc = 0.0
            for d in range(128):
                acc += float(q[r][d]) * float(k[j][d])
            s.append(acc * qd * kd / math.sqrt(128.0))
        mx = max(s)
        w = [math.exp(x - mx) for x in s]
        tot = sum(w)
        row = []
        for d in range(128):
            acc = 0.0
            for j in range(len(k)):
                acc += w[j] * float(v[j][d])
            row.append(acc / tot * vd)
        out.append(row)
        lse.append(mx + math.log(tot))
    return np.array(out), np.array(lse)


def test_brute_force_tiny_asymmetric():
    g = np.random.default_rng(3)
    q = g.standard_normal((3, 128)) * 2
    k = g.standard_normal((5, 128)) * 1.5 + 0.3
    v = g.standard_normal((5, 128)) - 0.2
    o, lse = oatt.attend_block(q, k, v, qd=0.75, kd=1.25, vd=2.0)
    ob, lb = _brute_attention(q, k, v, 0.75, 1.25, 2.0)
    assert np.allclose(o, ob, atol=1e-12, rtol=1e-12)
    assert np.allclose(lse, lb, atol=1e-12, rtol=1e-12)
    s = (q @ k.T) * 0.75 * 1.25 * SCALE
    assert np.allclose(lse, logsumexp(s, axis=1), atol=1e-12)


def test_varlen_packing_equals_separate_and_cross_pairing():
    g = np.random.default_rng(4)
    lq, lk = [3, 9, 1], [4, 2, 11]
    H = 2
    q = g.standard_normal((sum(lq), H, 128))
    k = g.standard_normal((sum(lk), H, 128))
    v = g.standard_normal((sum(lk), H, 128))
    o, lse = oatt.attention_fwd(q, k, v, lq, lk)
    assert lse.shape == (H, sum(lq))
    cq, ck = np.cumsum([0] + lq), np.cumsum([0] + lk)
    for i in range(3):
        for h in range(H):
            ob, lb = _brute_attention(q[cq[i]:cq[i + 1], h], k[ck[i]:ck[i + 1], h], v[ck[i]:ck[i + 1], h])
            assert np.allclose(o[cq[i]:cq[i + 1], h], ob, atol=1e-12)
            assert np.allclose(lse[h, cq[i]:cq[i + 1]], lb, atol=1e-12)


def test_key_permutation_invariance():
    g = np.random.default_rng(5)
    q, k, v = g.standard_normal((6, 128)), g.standard_normal((40, 128)), g.standard_normal((40, 128))
    perm = g.permutation(40)
    o1, l1 = oatt.attend_block(q, k, v)
    o2, l2 = oatt.attend_block(q, k[perm], v[perm])
    assert np.allclose(o1, o2, atol=1e-12) and np.allclose(l1, l2, atol=1e-12)


def test_descale_two_equals_scale_bytes_plus_one():
    """A q descale of 2 is the same as every Q scale byte raised by one."""
    g = np.random.default_rng(6)
    lens = [200]
    x = g.standard_normal((200, 2, 128)).astype(np.float32)
    kx = g.standard_normal((200, 2, 128)).astype(np.float32)
    vx = g.standard_normal((200, 2, 128)).astype(np.float32)
    pq, sq = omx.quantize_mxfp8_varlen(x, lens)
    pk, sk = omx.quantize_mxfp8_varlen(kx, lens)
    pv, sv = omx.quantize_mxfp8_varlen(vx, lens)
    kh = omx.dequantize_mxfp8(pk, sk, lens, 2)
    vh = omx.dequantize_mxfp8(pv, sv, lens, 2)
    qh = omx.dequantize_mxfp8(pq, sq, lens, 2)
    qh2 = omx.dequantize_mxfp8(pq, sq + np.uint8(1), lens, 2)
    assert np.allclose(qh2, 2 * qh, atol=0)
    o1, l1 = oatt.attention_fwd(qh, kh, vh, lens, lens, qd=2.0)
    o2, l2 = oatt.attention_fwd(qh2, kh, vh, lens, lens)
    assert np.allclose(o1, o2, atol=1e-12) and np.allclose(l1, l2, atol=1e-12)
    o3, _ = oatt.attention_fwd(qh, kh, vh, lens, lens)
    assert not np.allclose(o1, o3, atol=1e-3)


def _raise_scale_bytes(scales, lengths, heads, exps):
    """Scale storage with the bytes of (sequence i, head h) raised by exps[i, h]."""
    from oracle import meta as omt
    m = omt.from_lengths(lengths)
    out = scales.copy().reshape(-1, heads, 512)
    for i in range(m.num_seqs):
        for h in range(heads):
            out[m.scale_off[i]:m.scale_off[i + 1], h, :] += np.uint8(exps[i, h])
    return out.reshape(scales.shape)


def test_per_head_and_per_sequence_descales_equal_raised_scale_bytes():
    """vLLM PR #63232 ("Claims"): per-head scales keep their descale tensors. A per-head q descale
    of 2^e_h is the same as raising head h's Q scale bytes by e_h, and an (S, H) k descale of
    2^e_ih the same as raising the K bytes of sequence i, head h by e_ih; v descales scale O only."""
    g = np.random.default_rng(9)
    lens_q, lens_k, H = [150, 70], [90, 200], 3
    x = g.standard_normal((sum(lens_q), H, 128)).astype(np.float32)
    kx = g.standard_normal((sum(lens_k), H, 128)).astype(np.float32)
    vx = g.standard_normal((sum(lens_k), H, 128)).astype(np.float32)
    pq, sq = omx.quantize_mxfp8_varlen(x, lens_q)
    pk, sk = omx.quantize_mxfp8_varlen(kx, lens_k)
    pv, sv = omx.quantize_mxfp8_varlen(vx, lens_k)
    qh = omx.dequantize_mxfp8(pq, sq, lens_q, H)
    kh = omx.dequantize_mxfp8(pk, sk, lens_k, H)
    vh = omx.dequantize_mxfp8(pv, sv, lens_k, H)
    eq = np.array([1, -1, 2])
    ek = np.array([[0, 1, -2], [2, 0, 1]])
    qh2 = omx.dequantize_mxfp8(pq, _raise_scale_bytes(sq, lens_q, H, np.tile(eq, (2, 1))), lens_q, H)
    kh2 = omx.dequantize_mxfp8(pk, _raise_scale_bytes(sk, lens_k, H, ek), lens_k, H)
    o1, l1 = oatt.attention_fwd(qh, kh, vh, lens_q, lens_k, qd=2.0 ** eq, kd=2.0 ** ek)
    o2, l2 = oatt.attention_fwd(qh2, kh2, vh, lens_q, lens_k)
    assert np.allclose(o1, o2, atol=1e-12) and np.allclose(l1, l2, atol=1e-12)
    # a per-head v descale multiplies that head's O and leaves the LSE alone
    vd = np.array([1.0, 4.0, 0.5])
    o3, l3 = oatt.attention_fwd(qh, kh, vh, lens_q, lens_k, vd=vd.reshape(1, 3))
    o0, l0 = oatt.attention_fwd(qh, kh, vh, lens_q, lens_k)
    assert np.allclose(o3, o0 * vd[None, :, None], atol=1e-12) and np.array_equal(l3, l0)
    # broadcasting: (1, 1), (1,) and scalar are the same per-tensor value
    for d in (np.array([[2.0]]), np.array([2.0]), 2.0):
        o4, l4 = oatt.attention_fwd(qh, kh, vh, lens_q, lens_k, qd=d)
        o5, l5 = oatt.attention_fwd(qh, kh, vh, lens_q, lens_k, qd=2.0)
        assert np.array_equal(o4, o5) and np.array_equal(l4, l5)


def test_descale_at_indexing():
    d = np.arange(6, dtype=np.float64).reshape(2, 3)
    assert oatt.descale_at(d, 1, 2) == 5.0 and oatt.descale_at(d, 0, 1) == 1.0
    assert oatt.descale_at(np.array([7.0, 8.0, 9.0]), 1, 2) == 9.0
    assert oatt.descale_at(np.array([[3.0, 4.0]]), 1, 1) == 4.0   # size-1 sequence axis broadcasts
    assert oatt.descale_at(np.array([[3.0], [4.0]]), 1, 1) == 4.0  # size-1 head axis broadcasts
    assert oatt.descale_at(1.5, 3, 3) == 1.5


def test_fp8_variant_equals_plain_when_weights_exact():
    """Logits whose log2 values are integers give E4M3-exact weights: variant == definition."""
    g = np.random.default_rng(7)
    n = 24
    ints = g.integers(-12, 1, size=n).astype(np.float64)
    ints[3] = 0.0
    # s_j = ints_j * ln 2 through a single query q = e_0 and keys k_j = (c_j, 0, ...)
    q = np.zeros((1, 128)); q[0, 0] = 1.0
    k = np.zeros((n, 128)); k[:, 0] = ints * math.log(2.0) * math.sqrt(128.0)
    v = g.standard_normal((n, 128))
    o_plain, l_plain = oatt.attend_block(q, k, v, p_mode="exact")
    o_fp8, l_fp8 = oatt.attend_block(q, k, v, p_mode="fp8")
    assert np.allclose(o_plain, o_fp8, atol=1e-12)
    assert np.allclose(l_plain, l_fp8, atol=1e-12)


def test_fp8_variant_shift_invariance_and_brute_force():
    g = np.random.default_rng(8)
    q, k, v = g.standard_normal((3, 128)), g.standard_normal((50, 128)), g.standard_normal((50, 128))
    o1, _ = oatt.attend_block(q, k, v, p_mode="fp8")
    # shifting every logit of a row by 3*ln2 (via descale on a constant extra channel)
    qs = np.concatenate([q[:, :127], np.full((3, 1), 1.0)], axis=1)
    ks = np.concatenate([k[:, :127], np.full((50, 1), 3 * math.log(2) * math.sqrt(128.0))], axis=1)
    ob, _ = oatt.attend_block(qs, ks, v, p_mode="fp8")
    ks0 = np.concatenate([k[:, :127], np.zeros((50, 1))], axis=1)
    oa, _ = oatt.attend_block(qs, ks0, v, p_mode="fp8")
    assert np.allclose(oa, ob, atol=1e-12)
    # brute force with nearest-search rounding of 2^8 * 2^(t - ceil(max t))
    vals = omx.e4m3_decode_table()
    finite = [(c, vals[c]) for c in range(0x7F)]
    for r in range(3):
        t = [(q[r] @ k[j]) / math.sqrt(128) / math.log(2) for j in range(50)]
        ms = math.ceil(max(t))
        num = np.zeros(128)
        den = 0.0
        for j in range(50):
            u = 2.0 ** (t[j] - ms)
            den += u
            target = 256.0 * u
            best = min(finite, key=lambda cv: (abs(cv[1] - target), cv[0] % 2))
            num += best[1] / 256.0 * v[j]
        assert np.allclose(o1[r], num / den, atol=1e-12)


def test_fp8_variant_differs_from_plain_on_random_logits():
    """Negative control: the E4M3 rounding of P is visible on random inputs."""
    g = np.random.default_rng(9)
    q, k, v = g.standard_normal((64, 128)), g.standard_normal((512, 128)), g.standard_normal((512, 128))
    o1, _ = oatt.attend_block(q, k, v, p_mode="exact")
    o2, _ = oatt.attend_block(q, k, v, p_mode="fp8")
    rel = np.linalg.norm(o1 - o2) / np.linalg.norm(o1)
    assert 1e-3 < rel < 0.1


def test_attention_rows_matches_full():
    g = np.random.default_rng(10)
    lq, lk = [5, 7], [9, 3]
    q = g.standard_normal((12, 2, 128)); k = g.standard_normal((12, 2, 128)); v = g.standard_normal((12, 2, 128))
    o, lse = oatt.attention_fwd(q, k, v, lq, lk)
    rows = [0, 4, 5, 11]
    seqs = [0, 0, 1, 1]
    heads = [1, 0, 1, 0]
    orow, lrow = oatt.attention_rows(q[rows, heads], seqs, heads, k, v, lk)
    for i, (r, h) in enumerate(zip(rows, heads)):
        assert np.allclose(orow[i], o[r, h], atol=1e-12)
        assert np.isclose(lrow[i], lse[h, r], atol=1e-12)


def test_mxfp8_variant_equals_plain_when_weights_exact():
    """Weights that are powers of two within one E4M3 scale range of their group maximum are exact
    MXFP8 values: the block-scaled variant equals the plain definition."""
    g = np.random.default_rng(41)
    n = 70
    ints = g.integers(-14, 1, size=n).astype(np.float64)
    ints[[3, 40, 66]] = 0.0                                      # every 32-key group holds a 2^0
    q = np.zeros((1, 128)); q[0, 0] = 1.0
    k = np.zeros((n, 128)); k[:, 0] = ints * math.log(2.0) * math.sqrt(128.0)
    v = g.standard_normal((n, 128))
    o_plain, l_plain = oatt.attend_block(q, k, v, p_mode="exact")
    o_mx, l_mx = oatt.attend_block(q, k, v, p_mode="mxfp8")
    assert np.allclose(o_plain, o_mx, atol=1e-12) and np.allclose(l_plain, l_mx, atol=1e-12)


def test_mxfp8_variant_shift_invariance_and_brute_force():
    g = np.random.default_rng(42)
    q, k, v = g.standard_normal((3, 128)), g.standard_normal((75, 128)) * 2, g.standard_normal((75, 128))
    o1, _ = oatt.attend_block(q, k, v, p_mode="mxfp8")
    qs = np.concatenate([q[:, :127], np.full((3, 1), 1.0)], axis=1)
    ks = np.concatenate([k[:, :127], np.full((75, 1), 5 * math.log(2) * math.sqrt(128.0))], axis=1)
    ks0 = np.concatenate([k[:, :127], np.zeros((75, 1))], axis=1)
    oa, _ = oatt.attend_block(qs, ks0, v, p_mode="mxfp8")
    ob, _ = oatt.attend_block(qs, ks, v, p_mode="mxfp8")
    assert np.allclose(oa, ob, atol=1e-12)
    # brute force: per 32-key group, the smallest e with max u <= 448 * 2^e by search, and
    # nearest-value rounding (ties to even code) of u * 2^-e over the E4M3 table
    vals = omx.e4m3_decode_table()
    finite = [(c, vals[c]) for c in range(0x7F)]
    for r in range(3):
        t = [(q[r] @ k[j]) / math.sqrt(128) / math.log(2) for j in range(75)]
        ms = math.ceil(max(t))
        u = [2.0 ** (tj - ms) for tj in t]
        num = np.zeros(128)
        for g0 in range(0, 75, 32):
            grp = range(g0, min(75, g0 + 32))
            amax = max(u[j] for j in grp)
            e = next(e for e in range(-140, 20) if amax <= 448.0 * 2.0 ** e)
            for j in grp:
                best = min(finite, key=lambda cv: (abs(cv[1] - u[j] * 2.0 ** -e), cv[0] % 2))
                num += best[1] * 2.0 ** e * v[j]
        assert np.allclose(o1[r], num / sum(u), atol=1e-12)


def test_mxfp8_variant_differs_from_fp8_and_plain():
    """Where a 32-key group's weights are far below the row maximum, the per-group scale keeps
    their precision, while the fp8 variant's single power-of-two reference leaves them in the
    E4M3 subnormal range: one key at t = -15.3 is 256 * 2^-15.3 = 3.25 * 2^-9 there (rounded to
    3 * 2^-9, -7.7 %), but 1.625 * 2^-16 (exact to 0.03 %) under its own group scale."""
    t = np.full(64, -40.0)
    t[0] = 0.0                                          # group 0: the row maximum
    t[40] = -15.3                                       # group 1: a single small weight
    q = np.zeros((1, 128)); q[0, 0] = 1.0
    k = np.zeros((64, 128)); k[:, 0] = t * math.log(2.0) * math.sqrt(128.0)
    v = np.zeros((64, 128)); v[40, 1] = 1.0             # channel 1 sees key 40 only
    o_e, _ = oatt.attend_block(q, k, v, p_mode="exact")
    o_f, _ = oatt.attend_block(q, k, v, p_mode="fp8")
    o_m, _ = oatt.attend_block(q, k, v, p_mode="mxfp8")
    err_m = abs(o_m[0, 1] - o_e[0, 1]) / o_e[0, 1]
    err_f = abs(o_f[0, 1] - o_e[0, 1]) / o_e[0, 1]
    assert err_m < 2 ** -10 and 0.07 < err_f < 0.08, (err_m, err_f)


def test_shared_query_blocks_by_brute_force_and_closed_forms():
    """Shared-query reading (LP-FA4 README, opening paragraph: "shared-query workloads"): block i
    of the output is the attention of the one query set over key/value sequence i. Pinned by
    pure-Python brute force per block (with per-(sequence, head) descales), identical key/value
    sequences giving identical blocks, constant V giving V, and a single key giving that V row
    with LSE equal to its logit."""
    g = np.random.default_rng(21)
    Lq, H, lk = 3, 2, [4, 1, 6]
    q = g.standard_normal((Lq, H, 128))
    k = g.standard_normal((sum(lk), H, 128))
    v = g.standard_normal((sum(lk), H, 128))
    qd = np.array([0.5, 2.0])
    kd = np.array([[1.0, 0.5], [1.5, 1.0], [0.25, 3.0]])
    vd = 1.5
    o, lse = oatt.attention_fwd_shared_q(q, k, v, lk, qd, kd, vd)
    assert o.shape == (len(lk) * Lq, H, 128) and lse.shape == (H, len(lk) * Lq)
    cu = np.concatenate([[0], np.cumsum(lk)])
    for i in range(len(lk)):
        for h in range(H):
            ob, lb = _brute_attention(q[:, h], k[cu[i]:cu[i + 1], h], v[cu[i]:cu[i + 1], h], qd[h], kd[i, h], vd)
            assert np.allclose(o[i * Lq:(i + 1) * Lq, h], ob, atol=1e-12)
            assert np.allclose(lse[h, i * Lq:(i + 1) * Lq], lb, atol=1e-12)
    # single key (sequence 1): O = vd * v, LSE = that logit
    s1 = (q[:, 0] @ k[cu[1], 0]) * qd[0] * kd[1, 0] * SCALE
    assert np.allclose(o[Lq:2 * Lq, 0], vd * v[cu[1], 0][None], atol=1e-12)
    assert np.allclose(lse[0, Lq:2 * Lq], s1, atol=1e-12)
    # identical key/value sequences give identical blocks; constant V gives V
    k2 = np.concatenate([k[:4], k[:4]])
    v2 = np.concatenate([np.repeat(v[:1], 4, axis=0), np.repeat(v[:1], 4, axis=0)])
    o2, l2 = oatt.attention_fwd_shared_q(q, k2, v2, [4, 4])
    assert np.array_equal(o2[:Lq], o2[Lq:]) and np.array_equal(l2[:, :Lq], l2[:, Lq:])
    assert np.allclose(o2, np.broadcast_to(v[0][None], o2.shape), atol=1e-12)
