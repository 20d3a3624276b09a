"""Packed variable-length metadata (oracle side).

LP-FA4 README, section "MXFP8 forward and backward": inputs are packed
``(tokens, heads, 128)`` tensors described by one length per sequence, and each
sequence receives independent scale storage padded to a multiple of 128 tokens.
``Mxfp8VarlenMeta.from_lengths`` builds that description from a list of lengths.

Readings taken here (pages silent):
* lengths must be positive; a zero or negative length is an error;
* scale storage is counted in 128-token blocks: sequence i owns blocks
  ``[scale_off[i], scale_off[i+1])`` with ``scale_off[i+1] - scale_off[i] = ceil(len_i / 128)``;
* the number of 128-row query tiles of sequence i is the same ``ceil(len_i / 128)``.

Parity: pinned by tests against hand-computed prefix sums.
"""
from __future__ import annotations

import dataclasses

import numpy as np

BLOCK_TOKENS = 128


@dataclasses.dataclass
class VarlenMeta:
    lengths: np.ndarray        # (n,) int64
    cu_seqlens: np.ndarray     # (n+1,) int64, token offsets of each sequence
    scale_off: np.ndarray      # (n+1,) int64, offsets in 128-token scale blocks
    num_seqs: int
    total_tokens: int
    total_scale_blocks: int
    max_seqlen: int


def from_lengths(lengths) -> VarlenMeta:
    lens = [int(x) for x in lengths]
    if len(lens) == 0:
        raise ValueError("at least one sequence is required")
    for x in lens:
        if x <= 0:
            raise ValueError("sequence lengths must be positive")
    cu = [0]
    so = [0]
    for x in lens:
        cu.append(cu[-1] + x)
        so.append(so[-1] + (x + BLOCK_TOKENS - 1) // BLOCK_TOKENS)
    return VarlenMeta(
        lengths=np.array(lens, dtype=np.int64),
        cu_seqlens=np.array(cu, dtype=np.int64),
        scale_off=np.array(so, dtype=np.int64),
        num_seqs=len(lens),
        total_tokens=cu[-1],
        total_scale_blocks=so[-1],
        max_seqlen=max(lens),
    )
