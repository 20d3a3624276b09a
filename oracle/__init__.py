"""CPU oracle for the MXFP8 attention forward path (test infrastructure only).

This package is the slow, plain reference the CUDA library is checked against.
Only the tests, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / reference
arm of ``bench.py`` use it; the library never imports, links or calls it, and
it shares no code with the library (its inputs come from ``workloads``).

Everything is numpy in float64 (or exact integer arithmetic):

* ``meta``      -- packed varlen offsets and the 128-token-padded scale offsets
                   (LP-FA4 README, "MXFP8 forward and backward").
* ``mxfp8``     -- the E4M3 and E8M0 codecs, the RCEIL / FLOOR scale rules, the
                   quantizer with its scale-factor storage, and the unscaled E4M3
                   cast of V (FastVideo PR #1654, description).
* ``attention`` -- noncausal softmax(Q K^T / sqrt(128)) V with natural-log LSE,
                   per-tensor descales (vLLM PR #63232, "Claims"), and the
                   grading variant for the fp8 PV mode.

Parity status of each function is stated in its module header.
"""
from . import meta, mxfp8, attention  # noqa: F401
