"""Attention forward parity on the GPU against the fp64 oracle.

Tolerances: O max-abs 2e-2 and rel-L2 1e-2 (oracle before BF16 rounding), LSE max-abs 1e-3.
bf16 PV mode is compared with the plain definition; fp8 PV mode with the oracle's fp8-P
grading variant (P rounded to E4M3 against a power-of-two reference).
"""
import math

import numpy as np
import pytest
import torch

import workloads as wl
from oracle import attention as oatt
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import precision_attention_forward_b200 as lp


def _status_ok():
    st, detail = lp.lpfa_device_status()
    assert st == lp.LPFA_OK, f"device status {st} (site {detail})"


CASES = [
    # (lens_q, lens_k, heads)
    ([1], [1], 1),
    ([5], [5], 2),
    ([128], [128], 2),
    ([129], [129], 1),
    ([256], [256], 2),
    ([300, 77, 1], [300, 77, 1], 3),
    ([200], [1000], 2),                 # cross attention, several KV tiles
    ([64, 700], [513, 129], 2),         # cross varlen with ragged tails
]


@pytest.mark.parametrize("pv_mode", ["bf16", "fp8", "bf16v", "mxfp8"])
@pytest.mark.parametrize("case", range(len(CASES)))
def test_attention_small_cases(pv_mode, case):
    lq, lk, H = CASES[case]
    q, k, v = wl.small_random(100 + case, lq, lk, H)
    if pv_mode == "fp8":
        v = v * np.float32(2.0)
    o, lse = gu.run_path(lp, q, k, v, lq, lk, H, pv_mode=pv_mode)
    _status_ok()
    o_ref, lse_ref = gu.oracle_full(q, k, v, lq, lk, H, pv_mode=pv_mode)
    gu.assert_within(gu.compare_attention(o, lse, o_ref, lse_ref), f"{pv_mode} {lq}/{lk} H={H}")


@pytest.mark.parametrize("nseq", [200, 300])   # longest-first order (<= 256 sequences) and plain order
def test_many_sequences(nseq):
    g = np.random.default_rng(nseq)
    lq = g.integers(1, 300, size=nseq).tolist()
    lk = g.integers(1, 300, size=nseq).tolist()
    q, k, v = wl.small_random(31, lq, lk, 1)
    o, lse = gu.run_path(lp, q, k, v, lq, lk, 1, pv_mode="fp8")
    _status_ok()
    o_ref, lse_ref = gu.oracle_full(q, k, v, lq, lk, 1, pv_mode="fp8")
    gu.assert_within(gu.compare_attention(o, lse, o_ref, lse_ref), f"{nseq} sequences")


def test_attention_fp32_inputs():
    lq = lk = [333]
    q, k, v = wl.small_random(7, lq, lk, 2, dtype="fp32")
    o, lse = gu.run_path(lp, q, k, v, lq, lk, 2, in_dtype="fp32")
    o_ref, lse_ref = gu.oracle_full(q, k, v, lq, lk, 2)
    gu.assert_within(gu.compare_attention(o, lse, o_ref, lse_ref), "fp32 inputs")


@pytest.mark.parametrize("pv_mode", ["bf16", "fp8", "bf16v", "mxfp8"])
def test_closed_forms(pv_mode):
    """Constant V gives V (bf16 PV) or V times one scalar per row (fp8 PV, where l sums the
    unrounded weights); equal logits give LSE = ln n + s and O = the mean of V."""
    H, n = 2, 300
    g = np.random.default_rng(3)
    q = wl.round_to_bf16(g.standard_normal((n, H, 128)).astype(np.float32))
    krow = wl.round_to_bf16(g.standard_normal((1, H, 128)).astype(np.float32))
    k = np.repeat(krow, n, axis=0)
    v = wl.round_to_bf16(g.standard_normal((n, H, 128)).astype(np.float32))
    vconst = np.repeat(v[:1], n, axis=0)
    krand = wl.round_to_bf16(g.standard_normal((n, H, 128)).astype(np.float32))
    # constant V (random keys)
    o, lse = gu.run_path(lp, q, krand, vconst, [n], [n], H, pv_mode=pv_mode)
    qh, kh, vh = gu.oracle_inputs(q, krand, vconst, [n], [n], H, pv_mode)
    o_np = o.float().cpu().numpy().astype(np.float64)
    if pv_mode not in ("fp8", "mxfp8"):   # P rounded to 8 bits, l the unrounded sum: a ratio
        assert np.max(np.abs(o_np - vh[:1])) <= gu.O_MAX_ABS
    else:
        ratio = (o_np * vh[:1]).sum(axis=2) / (vh[:1] ** 2).sum(axis=2)      # (n, H)
        assert np.all(np.abs(ratio - 1.0) < 0.02)
        assert np.max(np.abs(o_np - ratio[..., None] * vh[:1])) <= gu.O_MAX_ABS
    # equal logits: all keys identical
    o, lse = gu.run_path(lp, q, k, v, [n], [n], H, pv_mode=pv_mode)
    qh, kh, vh = gu.oracle_inputs(q, k, v, [n], [n], H, pv_mode)
    s = np.einsum("thd,hd->ht", qh, kh[0]) / math.sqrt(128)
    assert np.max(np.abs(lse.cpu().numpy() - (np.log(n) + s))) < gu.LSE_MAX_ABS
    if pv_mode not in ("fp8", "mxfp8"):
        assert np.max(np.abs(o.float().cpu().numpy() - vh.mean(axis=0)[None])) <= gu.O_MAX_ABS


def test_single_key():
    q, k, v = wl.small_random(5, [77], [1], 2)
    o, lse = gu.run_path(lp, q, k, v, [77], [1], 2)
    qh, kh, vh = gu.oracle_inputs(q, k, v, [77], [1], 2)
    assert np.max(np.abs(o.float().cpu().numpy() - vh[:1])) <= gu.O_MAX_ABS
    s = np.einsum("thd,hd->ht", qh, kh[0]) / math.sqrt(128)
    assert np.max(np.abs(lse.cpu().numpy() - s)) < gu.LSE_MAX_ABS


@pytest.mark.parametrize("pv_mode", ["bf16", "fp8", "bf16v", "mxfp8"])
def test_unit_descale_is_bit_identical_and_two_changes_output(pv_mode):
    """vLLM #63232 'Validation': absent descale == unit descale bit for bit; 2 changes it."""
    w = wl.WORKLOADS["dense_4x2048_h16"]
    lq, lk = wl.lengths(w)
    q, k, v = (wl.make_tensor(w, x) for x in "qkv")
    if pv_mode == "fp8":
        v = v * np.float32(2.0)
    o0, l0 = gu.run_path(lp, q, k, v, lq, lk, w.heads, pv_mode=pv_mode)
    o1, l1 = gu.run_path(lp, q, k, v, lq, lk, w.heads, pv_mode=pv_mode, descales=(1.0, 1.0, 1.0))
    assert torch.equal(o0.view(torch.int16), o1.view(torch.int16))
    assert torch.equal(l0.view(torch.int32), l1.view(torch.int32))
    o2, l2 = gu.run_path(lp, q, k, v, lq, lk, w.heads, pv_mode=pv_mode, descales=(2.0, 1.0, 1.0))
    assert not torch.equal(o0, o2) and not torch.equal(l0, l2)
    o3, l3 = gu.run_path(lp, q, k, v, lq, lk, w.heads, pv_mode=pv_mode, descales=(1.0, 1.0, 2.0))
    assert not torch.equal(o0, o3)
    _status_ok()


@pytest.mark.parametrize("descales", [(2.0, 1.0, 1.0), (0.5, 3.0, 0.25), (-1.0, 1.0, 1.0), (1.0, 1.0, -2.0)])
def test_descale_values_match_oracle(descales):
    lq = lk = [400]
    q, k, v = wl.small_random(17, lq, lk, 2)
    o, lse = gu.run_path(lp, q, k, v, lq, lk, 2, descales=descales)
    o_ref, lse_ref = gu.oracle_full(q, k, v, lq, lk, 2, descales=descales)
    gu.assert_within(gu.compare_attention(o, lse, o_ref, lse_ref), f"descales {descales}")


@pytest.mark.parametrize("pv_mode", ["bf16", "fp8", "bf16v", "mxfp8"])
def test_per_head_and_per_sequence_descales_match_oracle(pv_mode):
    """vLLM #63232 'Claims': per-head scales keep their descale tensors. q (H,), k (S, H) and
    v (1, H) descales, with negative and non-power-of-two values, against the oracle."""
    # At least 64 keys per sequence: with a handful of keys, one E4M3 rounding decision of P that
    # falls differently in fp32 and fp64 moves O by more than the bound in fp8 PV mode, whatever
    # the descales (the few-key cases are covered without descales elsewhere).
    lq, lk, H = [300, 77, 129], [129, 700, 64], 3
    q, k, v = wl.small_random(31, lq, lk, H)
    if pv_mode == "fp8":
        v = v * np.float32(2)
    qd = np.array([0.5, -1.25, 2.0])
    kd = np.array([[1.0, 0.75, 3.0], [2.0, 1.0, -0.5], [0.25, 1.5, 1.0]])
    vd = np.array([[1.0, -2.0, 0.5]])
    o, lse = gu.run_path(lp, q, k, v, lq, lk, H, pv_mode=pv_mode, descales=(qd, kd, vd))
    o_ref, lse_ref = gu.oracle_full(q, k, v, lq, lk, H, pv_mode=pv_mode, descales=(qd, kd, vd))
    # The O bound is stated at unit output scale: a v descale multiplies O, and with it every
    # rounding error, exactly, so each head's O error is divided by |v descale| of that head.
    o_scale = np.abs(vd).reshape(1, H, 1)
    gu.assert_within(gu.compare_attention(o, lse, o_ref, lse_ref, o_scale=o_scale), f"per-head descales {pv_mode}")
    _status_ok()


@pytest.mark.parametrize("pv_mode", ["bf16", "fp8"])
def test_per_head_unit_descales_bit_identical_and_one_head_changes(pv_mode):
    """All-ones per-head descales == no descale bit for bit (vLLM #63232 'Validation'); a 2 on one
    head changes that head only; an expanded per-tensor view equals the per-tensor value."""
    lq = lk = [400, 200]
    H = 4
    q, k, v = wl.small_random(37, lq, lk, H)
    if pv_mode == "fp8":
        v = v * np.float32(2)
    o0, l0 = gu.run_path(lp, q, k, v, lq, lk, H, pv_mode=pv_mode)
    ones = np.ones(H)
    o1, l1 = gu.run_path(lp, q, k, v, lq, lk, H, pv_mode=pv_mode, descales=(ones, ones.reshape(1, H), ones))
    assert torch.equal(o0.view(torch.int16), o1.view(torch.int16))
    assert torch.equal(l0.view(torch.int32), l1.view(torch.int32))
    two_on_2 = np.array([1.0, 1.0, 2.0, 1.0])
    o2, l2 = gu.run_path(lp, q, k, v, lq, lk, H, pv_mode=pv_mode, descales=(two_on_2, None, None))
    for h in range(H):
        same_o = torch.equal(o0[:, h].view(torch.int16), o2[:, h].view(torch.int16))
        same_l = torch.equal(l0[h].view(torch.int32), l2[h].view(torch.int32))
        assert (same_o and same_l) == (h != 2), h
    # a per-tensor 2.0 given as a stride-0 (S, H) view equals the one-element tensor
    d1 = torch.tensor([2.0], dtype=torch.float32, device="cuda")
    o3, l3 = gu.run_path(lp, q, k, v, lq, lk, H, pv_mode=pv_mode, descales=(d1, None, d1))
    o4, l4 = gu.run_path(lp, q, k, v, lq, lk, H, pv_mode=pv_mode, descales=(d1.view(1, 1).expand(2, H), None,
                                                                          d1.expand(H)))
    assert torch.equal(o3.view(torch.int16), o4.view(torch.int16))
    assert torch.equal(l3.view(torch.int32), l4.view(torch.int32))
    _status_ok()


@pytest.mark.parametrize("pv_mode", ["fp8", "bf16", "bf16v", "mxfp8"])
def test_repeated_runs_are_bit_identical(pv_mode):
    """The kernel's result does not depend on timing: repeated calls on the same inputs give the
    same bits (a barrier phase completed by the wrong warps once made fp8 PV rows differ)."""
    w = wl.WORKLOADS["dense_4x2048_h16"]
    lq, lk = wl.lengths(w)
    q, k, v = (wl.make_tensor(w, x) for x in "qkv")
    if pv_mode == "fp8":
        v = v * np.float32(2.0)
    mq = lp.lpfa_varlen_meta_from_lengths(lq)
    mk = lp.lpfa_varlen_meta_from_lengths(lk)
    qp, qs = gu.gpu_quantize(lp, q, "bf16", mq)
    kp, ks = gu.gpu_quantize(lp, k, "bf16", mk)
    if pv_mode == "fp8":
        vp, vs = lp.lpfa_cast_e4m3(gu.to_device(v, "bf16")), None
    elif pv_mode == "bf16v":
        vp, vs = gu.to_device(v, "bf16"), None
    elif pv_mode == "mxfp8":
        vp, vs = lp.lpfa_quantize_mxfp8_varlen(gu.to_device(v, "bf16"), mk, orientation="tokens")
    else:
        vp, vs = gu.gpu_quantize(lp, v, "bf16", mk)
    ref = None
    for _ in range(4):
        o, lse = lp.lpfa_attn_fwd_varlen(qp, qs, kp, ks, vp, vs, mq, mk, pv_mode=pv_mode)
        torch.cuda.synchronize()
        if ref is None:
            ref = (o.clone(), lse.clone())
            continue
        assert torch.equal(o.view(torch.int16), ref[0].view(torch.int16))
        assert torch.equal(lse.view(torch.int32), ref[1].view(torch.int32))
    _status_ok()


def test_negative_control_wrong_k_scales_fail():
    """Scale bytes of K raised by one (K doubled) must fail the tolerance."""
    lq = lk = [512]
    q, k, v = wl.small_random(23, lq, lk, 2)
    mq = lp.lpfa_varlen_meta_from_lengths(lq)
    mk = lp.lpfa_varlen_meta_from_lengths(lk)
    qp, qs = gu.gpu_quantize(lp, q, "bf16", mq)
    kp, ks = gu.gpu_quantize(lp, k, "bf16", mk)
    vp, vs = gu.gpu_quantize(lp, v, "bf16", mk)
    o, lse = lp.lpfa_attn_fwd_varlen(qp, qs, kp, ks + 1, vp, vs, mq, mk)
    o_ref, lse_ref = gu.oracle_full(q, k, v, lq, lk, 2)
    max_abs, rel, lmax = gu.compare_attention(o, lse, o_ref, lse_ref)
    assert lmax > gu.LSE_MAX_ABS and rel > gu.O_REL_L2


@pytest.mark.parametrize("name", ["single_s256_h2", "dense_4x2048_h16", "dense_4x2048_h16_bf16v", "dense_4x2048_h16_mxpv"])
@pytest.mark.parametrize("mode", ["rceil", "floor"])
def test_workload_full_check(name, mode):
    w = wl.WORKLOADS[name]
    lq, lk = wl.lengths(w)
    q, k, v = (wl.make_tensor(w, x) for x in "qkv")
    o, lse = gu.run_path(lp, q, k, v, lq, lk, w.heads, in_dtype=w.in_dtype, pv_mode=w.pv_mode, mode=mode)
    _status_ok()
    o_ref, lse_ref = gu.oracle_full(q, k, v, lq, lk, w.heads, pv_mode=w.pv_mode, mode=mode)
    print(gu.assert_within(gu.compare_attention(o, lse, o_ref, lse_ref), f"{name} {mode}"))


@pytest.mark.slow
@pytest.mark.parametrize("name", ["varlen16_fp32_h16", "video_s32768_h24_fp8pv", "cross_varlen_outliers_h32",
                                  "video_s32768_h24_mxpv"])
def test_workload_sampled_check(name):
    """Full-size run in the benchmarked launch configuration, checked on sampled rows that
    cover every (sequence, head), each 128-row tile and every tail."""
    w = wl.WORKLOADS[name]
    lq, lk = wl.lengths(w)
    q, k, v = (wl.make_tensor(w, x) for x in "qkv")
    o, lse = gu.run_path(lp, q, k, v, lq, lk, w.heads, in_dtype=w.in_dtype, pv_mode=w.pv_mode)
    _status_ok()
    toks, hs = gu.sample_rows(lq, w.heads, seed=11, per_tile_random=0 if name.startswith("video") else 1)
    if name.startswith("video"):
        # 24 heads x 256 tiles: keep the oracle bounded to every 8th tile plus all edges.
        keep = (toks % 1024 < 128) | (toks == toks.max())
        toks, hs = toks[keep], hs[keep]
    o_ref, lse_ref = gu.oracle_sampled(q, k, v, lq, lk, w.heads, toks, hs, pv_mode=w.pv_mode)
    tt, hh = torch.from_numpy(toks).cuda(), torch.from_numpy(hs).cuda()
    o_s = o[tt, hh]
    lse_s = lse[hh, tt]
    o_scale = wl.outlier_scale(w, "v")[hs] if w.outlier_frac > 0.0 else None
    print(gu.assert_within(gu.compare_attention(o_s, lse_s, o_ref, lse_ref, o_scale), f"{name} sampled"))


def _rising_inputs(seed, lq, lk, H):
    """Q and K whose logits jump by about 9 binades (times a per-row slope in [0.5, 1.5]) from each
    128-key tile to the next, through one spike key per tile; V random.

    The jump exceeds the softmax reference's lag in every mode (2 binades for fp8 P, 8 otherwise)
    for most rows, so the kernel moves the row reference and rescales O on almost every tile,
    while the earlier tiles keep a share of the weight that a missing or wrong rescale would
    visibly change. Logits in log2 units are a_r * level(key) + noise, with level = 9 (t - 1)
    for the keys of tile t >= 1 and one key per tile at level + 9."""
    g = np.random.default_rng(seed)
    c = math.sqrt(math.log(2.0) * math.sqrt(128.0))     # (c u).(c u) / sqrt(128) = ln 2
    u = g.standard_normal((H, 128))
    u /= np.linalg.norm(u, axis=1, keepdims=True)
    q_rows, k_rows = [], []
    for n in lq:
        a = g.uniform(0.5, 1.5, size=(n, H, 1))
        q_rows.append(a * c * u[None] + 0.05 * g.standard_normal((n, H, 128)))
    for n in lk:
        tile = np.arange(n) // 128
        level = np.where(tile >= 1, 9.0 * (tile - 1), 0.0)
        spike = (np.arange(n) % 128 == 37) & (tile >= 1)
        level = level + 9.0 * spike
        k_rows.append(level[:, None, None] * c * u[None] + 0.5 * g.standard_normal((n, H, 128)))
    q = wl.round_to_bf16(np.concatenate(q_rows).astype(np.float32))
    k = wl.round_to_bf16(np.concatenate(k_rows).astype(np.float32))
    v = wl.round_to_bf16(g.standard_normal((sum(lk), H, 128)).astype(np.float32))
    return q, k, v


@pytest.mark.parametrize("pv_mode", ["bf16", "fp8", "bf16v", "mxfp8"])
def test_reference_moves_rescale_o(pv_mode):
    """The online softmax's correction step: when a later key tile's logits exceed the row
    reference by more than the lag, O and l are rescaled by an exact power of two before that
    tile's P V is added (LP-FA4 README, "MXFP8 forward and backward": online-softmax forward).
    Both query tiles of a pair, a single last tile, and ragged key tails are covered."""
    lq, lk, H = [300, 256], [600, 520], 2
    q, k, v = _rising_inputs(41, lq, lk, H)
    if pv_mode == "fp8":
        v = v * np.float32(2.0)
    o, lse = gu.run_path(lp, q, k, v, lq, lk, H, pv_mode=pv_mode)
    _status_ok()
    o_ref, lse_ref = gu.oracle_full(q, k, v, lq, lk, H, pv_mode=pv_mode)
    gu.assert_within(gu.compare_attention(o, lse, o_ref, lse_ref), f"rising logits {pv_mode}")
    # The earlier tiles matter: dropping every tile but the last changes O beyond the bound, so
    # the comparison above sees a wrong rescale of the earlier contributions.
    qh, kh, vh = gu.oracle_inputs(q, k, v, lq, lk, H, pv_mode)
    last = []
    for i, (n, m) in enumerate(zip(lq, lk)):
        k0 = sum(lk[:i])
        t0 = (m - 1) // 128 * 128
        oo, _ = oatt.attention_fwd(qh[sum(lq[:i]):sum(lq[:i]) + n], kh[k0 + t0:k0 + m], vh[k0 + t0:k0 + m],
                                   [n], [m - t0], p_mode=gu.p_mode_of(pv_mode))
        last.append(oo)
    d = np.concatenate(last) - o_ref
    assert np.linalg.norm(d) / np.linalg.norm(o_ref) > 5 * gu.O_REL_L2


@pytest.mark.parametrize("pv_mode", ["bf16", "fp8"])
@pytest.mark.parametrize("lens", [[300] * 10, [512] * 10])
def test_split_tail_units(pv_mode, lens):
    """320 pair units on a 148-CTA grid leave 24 for a last partial wave; they run as 48 single-tile
    units. With 3-tile sequences some of those are the absent second tile of a pair (skipped)."""
    H = 16
    q, k, v = wl.small_random(7 + lens[0], lens, lens, H)
    if pv_mode == "fp8":
        v = v * np.float32(2.0)
    o, lse = gu.run_path(lp, q, k, v, lens, lens, H, pv_mode=pv_mode)
    _status_ok()
    o_ref, lse_ref = gu.oracle_full(q, k, v, lens, lens, H, pv_mode=pv_mode)
    gu.assert_within(gu.compare_attention(o, lse, o_ref, lse_ref), f"split tail {pv_mode} {lens[0]}")
