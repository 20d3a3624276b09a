"""Attention backward at the video shape (1 x 32768 queries and keys, 24 heads) on the GPU:
sampled rows against the oracle evaluated row by row (oracle/backward.py,
attend_block_backward_sampled). Kept apart from the small-case backward tests because it draws
about 1.6 GB of host inputs."""
import numpy as np
import pytest
import torch

import workloads as wl
from tests import gpu_util as gu
from tests.test_attention_bwd_gpu import _grad_close

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import precision_attention_forward_b200 as lp


def test_backward_video_shape_sampled():
    """The video shape (1 x 32768 queries and keys, 24 heads) as bench.py --pass bwd runs it: a
    bf16-PV forward on MXFP8 Q/K/V, then the backward with a seeded BF16 dO. Rows of dQ, dK and dV
    of the first and last head, at tile boundaries and both ends, against the oracle evaluated
    row by row from the definition (tests.gpu_util.sampled_backward_reference)."""
    w = wl.WORKLOADS["video_s32768_h24_fp8pv"]
    lq, lk = wl.lengths(w)
    q, k, v = (wl.make_tensor(w, x) for x in "qkv")
    mq = lp.lpfa_varlen_meta_from_lengths(lq)
    mk = lp.lpfa_varlen_meta_from_lengths(lk)
    qp, qs = gu.gpu_quantize(lp, q, "bf16", mq)
    kp, ks = gu.gpu_quantize(lp, k, "bf16", mk)
    vp, vs = gu.gpu_quantize(lp, v, "bf16", mk)
    o, lse = lp.lpfa_attn_fwd_varlen(qp, qs, kp, ks, vp, vs, mq, mk, pv_mode="bf16")
    g = np.random.default_rng(7)
    do = wl.round_to_bf16(g.standard_normal(q.shape, dtype=np.float32))
    dq, dk, dv = lp.lpfa_attn_bwd_varlen(qp, qs, kp, ks, vp, vs, o, gu.to_device(do, "bf16"), lse, mq, mk)
    torch.cuda.synchronize()
    assert lp.lpfa_device_status() == (lp.LPFA_OK, 0)
    n = int(lq[0])
    idx = [0, 1, 127, 128, 4097, 16383, 16384, n - 129, n - 1]
    ti = torch.tensor(idx, device=dq.device)
    o_host = o.float().cpu().numpy()
    lse_host = lse.cpu().numpy()
    for h in (0, w.heads - 1):
        rq, rk, rv = gu.sampled_backward_reference(q, k, v, o_host, do, lse_host, lq, lk, h, idx, idx)
        for name, got, ref in (("dQ", dq, rq), ("dK", dk, rk), ("dV", dv, rv)):
            _grad_close(got[ti, h].float().cpu().numpy(), ref, f"{name} head {h}")
