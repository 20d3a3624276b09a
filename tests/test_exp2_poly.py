"""The FMA-pipe exp2 used for part of the softmax: float32 emulation of its exact steps.

The kernel evaluates 2^x as 2^j * q(x - j) with j = round(x) taken from the low mantissa bits
of x + 1.5 * 2^23, and q a cubic fitted by csrc/exp2_poly_fit.py. This test replays those
float32 operations in numpy (no GPU) and checks the relative error against exact 2^x, and
that the constants compiled into the kernel are the fitted ones.
"""
import os
import re

import numpy as np

from precision_attention_forward_b200.csrc import exp2_poly_fit

CUH = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "precision_attention_forward_b200", "csrc", "attn_fwd.cuh")


def kernel_coefficients():
    text = open(CUH).read()
    vals = {}
    for k in range(4):
        m = re.search(r"kExp2P%d\s*=\s*([0-9.eE+-]+)f;" % k, text)
        vals[k] = np.float32(float(m.group(1)))
    return [vals[k] for k in range(4)]


def emulate(x, c):
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-126.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    jf = (t - magic).astype(np.float32)
    f = (x - jf).astype(np.float32)          # exact: x and jf are within 0.5
    q = (np.float32(c[3]) * f + np.float32(c[2])).astype(np.float32)
    q = (q * f + np.float32(c[1])).astype(np.float32)
    q = (q * f + np.float32(c[0])).astype(np.float32)
    bits = q.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(np.float32)


def test_kernel_constants_are_the_fit():
    fitted = exp2_poly_fit.fit(3).astype(np.float32)
    assert np.array_equal(np.array(kernel_coefficients(), dtype=np.float32), fitted)


def test_relative_error_over_range():
    c = kernel_coefficients()
    # Results stay normal floats for x >= -125 (q may be just below 1 at the -126 binade).
    x = np.concatenate([np.linspace(-125.0, 2.0, 2_000_001, dtype=np.float32),
                        np.arange(-125, 3, dtype=np.float32),            # integers
                        np.arange(-125, 2, dtype=np.float32) + 0.5])     # round-half cases
    got = emulate(x, c).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() < 1.0e-4, rel.max()
    assert exp2_poly_fit.rounded_error(np.array(c, dtype=np.float32)) < 1.0e-4


def test_clamp_gives_tiny_nonnegative():
    c = kernel_coefficients()
    got = emulate(np.array([-1e4, -300.0, -127.0, -126.4], dtype=np.float32), c)
    assert np.all(got >= 0) and np.all(got < 2.0 ** -125)
