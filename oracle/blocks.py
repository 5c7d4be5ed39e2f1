"""Block-by-block generation: encode & append.

[Report] "DiffusionGemma Technical Report", Figure 4: generation runs block
after block; each 256-slot canvas block starts from noise, is denoised by
the adaptive loop until it settles, and the finished block is then encoded
and appended to the context the next block is conditioned on.  The model
(its encoder and KV cache) is out of scope: the caller's ``hidden_fn`` stands
in for it and receives the blocks committed so far.  Every block draws its
own random streams: the block index enters the Philox counter's step word
(``step.counter_step``), and a block's starting canvas is uniform noise
(``step.initial_canvas``, [Report] Figure 3).

TEST INFRASTRUCTURE: part of the CPU oracle (see ``oracle/__init__``).
"""
from __future__ import annotations

from dataclasses import replace

import numpy as np

from .loop import denoise_loop
from .step import Params, initial_canvas


def generate_blocks(hidden_fn, *, n_blocks: int, E_bits=None, q=None, s=None, B: int, L: int = 256,
                    params: Params = Params()):
    """Generate ``n_blocks`` blocks of B canvases.

    ``hidden_fn(j, k, canvas, committed)`` returns the bf16 hidden-state bits
    [B*L, d] of step k of block j, given the block's current canvas [B*L]
    and the committed blocks 0..j-1 ([j, B*L]).  Block j is numbered
    ``params.block + j`` in the random streams.  Returns (committed blocks
    int32 [n_blocks, B*L], steps taken int32 [n_blocks, B]).
    """
    V = (E_bits if E_bits is not None else q).shape[0]
    blocks = np.zeros((n_blocks, B * L), np.int32)
    steps = np.zeros((n_blocks, B), np.int32)
    for j in range(n_blocks):
        pj = replace(params, block=params.block + j)
        canvas0 = np.concatenate([initial_canvas(b, pj.block, L, V, pj.seed) for b in range(B)])
        committed = blocks[:j].copy()
        fin, st, _ = denoise_loop(lambda k, c: hidden_fn(j, k, c, committed), E_bits=E_bits, q=q, s=s,
                                  B=B, L=L, params=pj, canvas=canvas0)
        blocks[j] = fin
        steps[j] = st
    return blocks, steps
