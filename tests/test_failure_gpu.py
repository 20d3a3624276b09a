"""Failure detection without a GPU fault, and out-of-bounds write detection.

* Bounded waits: the debug entry point makes the attention kernel's QK issuer wait on a barrier
  phase that never completes. The wait must run out (no hang), the kernel must record
  LPFA_ERR_TIMEOUT in the device status word, and the context must stay usable: a normal call
  right after gives the oracle's result.
* Guard bytes: every output buffer (payloads, scale storage, O, LSE) is a view into a larger
  buffer whose surrounding bytes hold a pattern; no kernel may touch them.
"""
import time

import numpy as np
import pytest
import torch

import workloads as wl
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import precision_attention_forward_b200 as lp

GUARD = 4096
PATTERN = 0xA5


def _guarded(nbytes: int):
    """A uint8 view of nbytes inside a buffer with GUARD pattern bytes on both sides."""
    buf = torch.full((nbytes + 2 * GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
    return buf, buf[GUARD:GUARD + nbytes]


def _guards_intact(buf: torch.Tensor, nbytes: int) -> bool:
    head = buf[:GUARD]
    tail = buf[GUARD + nbytes:]
    return bool(torch.all(head == PATTERN).item()) and bool(torch.all(tail == PATTERN).item())


@pytest.mark.parametrize("pv_mode", ["fp8", "bf16", "bf16v", "mxfp8"])
def test_bounded_wait_runs_out_and_context_survives(pv_mode):
    lens, H = [300, 77], 2
    q, k, v = wl.small_random(11, lens, lens, H)
    if pv_mode == "fp8":
        v = v * np.float32(2)
    mq = lp.lpfa_varlen_meta_from_lengths(lens)
    mk = lp.lpfa_varlen_meta_from_lengths(lens)
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
    assert lp.lpfa_device_status() == (lp.LPFA_OK, 0)

    t0 = time.time()
    lp.lpfa_attn_fwd_varlen(qp, qs, kp, ks, vp, vs, mq, mk, pv_mode=pv_mode, debug_flags=1)
    st, detail = lp.lpfa_device_status()
    elapsed = time.time() - t0
    assert st == lp.LPFA_ERR_TIMEOUT, (st, detail)
    assert detail != 0
    assert elapsed < 30.0, elapsed
    # The status word was reset by the read.
    assert lp.lpfa_device_status() == (lp.LPFA_OK, 0)

    o, lse = lp.lpfa_attn_fwd_varlen(qp, qs, kp, ks, vp, vs, mq, mk, pv_mode=pv_mode)
    torch.cuda.synchronize()
    assert lp.lpfa_device_status() == (lp.LPFA_OK, 0)
    ro, rl = gu.oracle_full(q, k, v, lens, lens, H, pv_mode=pv_mode)
    gu.assert_within(gu.compare_attention(o, lse, ro, rl), f"after timeout, {pv_mode}")


def test_unknown_debug_flag_rejected():
    lens, H = [5], 1
    q, k, v = wl.small_random(1, lens, lens, H)
    mq = lp.lpfa_varlen_meta_from_lengths(lens)
    qp, qs = gu.gpu_quantize(lp, q, "bf16", mq)
    kp, ks = gu.gpu_quantize(lp, k, "bf16", mq)
    vp, vs = gu.gpu_quantize(lp, v, "bf16", mq)
    with pytest.raises(lp.LpfaError) as e:
        lp.lpfa_attn_fwd_varlen(qp, qs, kp, ks, vp, vs, mq, mq, pv_mode="bf16", debug_flags=2)
    assert e.value.status == lp.LPFA_ERR_INVALID_ARG


@pytest.mark.parametrize("pv_mode", ["fp8", "bf16", "bf16v", "mxfp8"])
@pytest.mark.parametrize("lens_q,lens_k,H", [([1], [1], 1), ([300, 77, 1], [129, 700, 3], 3), ([2048], [257], 2)])
def test_outputs_stay_inside_their_buffers(pv_mode, lens_q, lens_k, H):
    q, k, v = wl.small_random(3, lens_q, lens_k, H)
    mq = lp.lpfa_varlen_meta_from_lengths(lens_q)
    mk = lp.lpfa_varlen_meta_from_lengths(lens_k)
    Tq, Tk = sum(lens_q), sum(lens_k)
    bufs = {}

    def alloc(name, nbytes):
        bufs[name] = _guarded(nbytes)
        return bufs[name][1]

    qp = alloc("qp", Tq * H * 128).view(Tq, H, 128)
    qs = alloc("qs", mq.scale_bytes(H))
    kp = alloc("kp", Tk * H * 128).view(Tk, H, 128)
    ks = alloc("ks", mk.scale_bytes(H))
    vp = gu.to_device(v, "bf16") if pv_mode == "bf16v" else alloc("vp", Tk * H * 128).view(Tk, H, 128)
    vs = alloc("vs", mk.scale_bytes(H)) if pv_mode in ("bf16", "mxfp8") else None
    out = alloc("out", Tq * H * 128 * 2).view(torch.bfloat16).view(Tq, H, 128)
    lse = alloc("lse", H * Tq * 4).view(torch.float32).view(H, Tq)

    lp.lpfa_quantize_mxfp8_varlen(gu.to_device(q, "bf16"), mq, payload=qp, scales=qs)
    lp.lpfa_quantize_mxfp8_varlen(gu.to_device(k, "bf16"), mk, payload=kp, scales=ks)
    if pv_mode == "fp8":
        lp.lpfa_cast_e4m3(gu.to_device(v, "bf16"), out=vp)
    elif pv_mode == "bf16":
        lp.lpfa_quantize_mxfp8_varlen(gu.to_device(v, "bf16"), mk, payload=vp, scales=vs)
    elif pv_mode == "mxfp8":
        lp.lpfa_quantize_mxfp8_varlen(gu.to_device(v, "bf16"), mk, payload=vp, scales=vs, orientation="tokens")
    lp.lpfa_attn_fwd_varlen(qp, qs, kp, ks, vp, vs, mq, mk, pv_mode=pv_mode, out=out, lse=lse)
    torch.cuda.synchronize()
    assert lp.lpfa_device_status() == (lp.LPFA_OK, 0)
    for name, (buf, view) in bufs.items():
        assert _guards_intact(buf, view.numel()), f"{name}: bytes outside the buffer were written"
    ro, rl = gu.oracle_full(q, k, v, lens_q, lens_k, H, pv_mode=pv_mode)
    gu.assert_within(gu.compare_attention(out, lse, ro, rl), f"guarded {pv_mode} {lens_q}/{lens_k}")


def _backward_inputs(lq, lk, H, seed):
    """MXFP8 Q/K/V, the forward's O and LSE, and a seeded dO on the device; the float inputs too."""
    q, k, v = wl.small_random(seed, lq, lk, H)
    g = np.random.default_rng(seed + 1000)
    do = wl.round_to_bf16(g.standard_normal((sum(lq), H, 128)).astype(np.float32))
    mq = lp.lpfa_varlen_meta_from_lengths(lq)
    mk = lp.lpfa_varlen_meta_from_lengths(lk)
    qp, qs = gu.gpu_quantize(lp, q, "bf16", mq)
    kp, ks = gu.gpu_quantize(lp, k, "bf16", mk)
    vp, vs = gu.gpu_quantize(lp, v, "bf16", mk)
    o, lse = lp.lpfa_attn_fwd_varlen(qp, qs, kp, ks, vp, vs, mq, mk, pv_mode="bf16")
    dev = (qp, qs, kp, ks, vp, vs, o, gu.to_device(do, "bf16"), lse, mq, mk)
    return dev, (q, k, v, do)


def _backward_reference(host, dev, lq, lk, H):
    from oracle import backward as obwd
    q, k, v, do = host
    o, lse = dev[6], dev[8]
    qh, kh, vh = gu.oracle_inputs(q, k, v, lq, lk, H)
    return obwd.attention_bwd(qh, kh, vh, o.float().cpu().numpy().astype(np.float64), do.astype(np.float64),
                              lse.cpu().numpy().astype(np.float64), lq, lk)


def _grads_close(got, ref):
    got = np.asarray(got, dtype=np.float64)
    rel = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-4 * np.sqrt(ref.size))
    mx = np.max(np.abs(got - ref)) / max(np.max(np.abs(ref)), 1e-4)
    return rel <= 1e-2 and mx <= 2e-2


def test_backward_bounded_wait_runs_out_and_context_survives():
    """The backward's waits are bounded like the forward's (LP-FA4 README, "MXFP8 forward and
    backward": mxfp8_flash_attn_varlen_backward): the debug hook makes the dK/dV kernel's MMA warp
    wait on a phase nothing completes; the call ends with LPFA_ERR_TIMEOUT in the status word and
    no fault, and a normal call right after matches the oracle."""
    lq, lk, H = [300, 77], [300, 77], 2
    dev, host = _backward_inputs(lq, lk, H, 21)
    torch.cuda.synchronize()
    assert lp.lpfa_device_status() == (lp.LPFA_OK, 0)
    t0 = time.time()
    lp.lpfa_attn_bwd_varlen(*dev, debug_flags=1)
    st, detail = lp.lpfa_device_status()
    elapsed = time.time() - t0
    assert st == lp.LPFA_ERR_TIMEOUT, (st, detail)
    assert 200 <= detail <= 207, detail
    assert elapsed < 30.0, elapsed
    assert lp.lpfa_device_status() == (lp.LPFA_OK, 0)
    dq, dk, dv = lp.lpfa_attn_bwd_varlen(*dev)
    torch.cuda.synchronize()
    assert lp.lpfa_device_status() == (lp.LPFA_OK, 0)
    for got, ref in zip((dq, dk, dv), _backward_reference(host, dev, lq, lk, H)):
        assert _grads_close(got.float().cpu().numpy(), ref)


def test_backward_unknown_debug_flag_rejected():
    dev, _ = _backward_inputs([5], [5], 1, 2)
    with pytest.raises(lp.LpfaError) as e:
        lp.lpfa_attn_bwd_varlen(*dev, debug_flags=2)
    assert e.value.status == lp.LPFA_ERR_INVALID_ARG


@pytest.mark.parametrize("mx_dkv", [False, True])
@pytest.mark.parametrize("lens_q,lens_k,H", [([1], [1], 1), ([300, 77, 1], [129, 700, 3], 3), ([2048], [257], 2)])
def test_backward_outputs_stay_inside_their_buffers(mx_dkv, lens_q, lens_k, H):
    """dQ, dK, dV and (MXFP8 output) the dK/dV scale storage, each inside pattern-filled guards."""
    dev, host = _backward_inputs(lens_q, lens_k, H, 5)
    Tq, Tk = sum(lens_q), sum(lens_k)
    mk = dev[10]
    bufs = {}

    def alloc(name, nbytes):
        bufs[name] = _guarded(nbytes)
        return bufs[name][1]

    dq = alloc("dq", Tq * H * 128 * 2).view(torch.bfloat16).view(Tq, H, 128)
    kv_bytes = Tk * H * 128 * (1 if mx_dkv else 2)
    kv_dtype = torch.uint8 if mx_dkv else torch.bfloat16
    dk = alloc("dk", kv_bytes).view(kv_dtype).view(Tk, H, 128)
    dv = alloc("dv", kv_bytes).view(kv_dtype).view(Tk, H, 128)
    extra = {}
    if mx_dkv:
        extra = {"dk_sf": alloc("dk_sf", mk.scale_bytes(H)), "dv_sf": alloc("dv_sf", mk.scale_bytes(H))}
    lp.lpfa_attn_bwd_varlen(*dev, output_mxfp8_dkv=mx_dkv, dq=dq, dk=dk, dv=dv, **extra)
    torch.cuda.synchronize()
    assert lp.lpfa_device_status() == (lp.LPFA_OK, 0)
    for name, (buf, view) in bufs.items():
        assert _guards_intact(buf, view.numel()), f"{name}: bytes outside the buffer were written"
    rq, rk, rv = _backward_reference(host, dev, lens_q, lens_k, H)
    assert _grads_close(dq.float().cpu().numpy(), rq)
    if not mx_dkv:
        assert _grads_close(dk.float().cpu().numpy(), rk) and _grads_close(dv.float().cpu().numpy(), rv)
    else:
        from oracle import mxfp8 as omx
        for pl, sc, ref in ((dk, extra["dk_sf"], rk), (dv, extra["dv_sf"], rv)):
            deq = omx.dequantize_mxfp8(pl.cpu().numpy(), sc.cpu().numpy(), lens_k, H)
            assert np.linalg.norm(deq - ref) <= 5e-2 * max(np.linalg.norm(ref), 1e-4 * np.sqrt(ref.size))
