"""The adaptive denoising loop over one block of canvases.

[Docs] "Recommended serving configuration": at most N = 48 steps per canvas;
stop early when the canvas-mean entropy is under 0.005 and two consecutive
predictions agree.  [Report] Figure 4: the denoising loop refines the canvas
until it is clean.  [Press] "What DiffusionGemma does": when the block has
settled, its still-open positions get fixed -- read here as: at the stopping
step (or the last allowed step) every slot takes that step's sampled token.
Each canvas stops on its own; a stopped canvas is frozen.

TEST INFRASTRUCTURE: part of the CPU oracle (see ``oracle/__init__``).
"""
from __future__ import annotations

import numpy as np

from .step import Params, denoise_step


def denoise_loop(hidden_fn, *, E_bits=None, q=None, s=None, B: int, L: int = 256,
                 params: Params = Params(), k_start: int = 0, canvas=None,
                 prev_argmax=None, has_prev=None, canvases=None):
    """Run steps k_start .. N-1 until every canvas stops.

    ``hidden_fn(k, canvas)`` returns the bf16 hidden-state bits [B*L, d] of
    step k.  Returns (final canvas int32 [B*L], steps taken int32 [B], the
    per-step history of stop flags and mean entropies).  With ``canvases``
    only those canvases of the batch are run (canvases are independent: each
    has its own random streams); the others keep their input canvas and 0
    steps.
    """
    N = params.max_steps
    V = (E_bits if E_bits is not None else q).shape[0]
    canvas = np.zeros(B * L, np.int32) if canvas is None else np.array(canvas, np.int32)
    prev = np.zeros(B * L, np.int32) if prev_argmax is None else np.array(prev_argmax, np.int32)
    hp = np.zeros(B, np.uint8) if has_prev is None else np.array(has_prev, np.uint8)
    active = np.zeros(B, dtype=bool)
    active[list(range(B)) if canvases is None else [int(c) for c in canvases]] = True
    steps = np.zeros(B, np.int32)
    history = []
    for k in range(k_start, N):
        h = hidden_fn(k, canvas)
        act = [b for b in range(B) if active[b]]
        r = denoise_step(h, E_bits=E_bits, q=q, s=s, B=B, L=L,
                         step_idx=np.full(B, k, np.int32), has_prev=hp,
                         prev_argmax=prev, params=params, canvases=act)
        history.append({"k": k, "canvases": act, "stop": r["stop"].copy(),
                        "mean_entropy": r["entropy"].reshape(len(act), L).mean(axis=1),
                        "n_accept": r["n_accept"].copy()})
        for i, b in enumerate(act):
            sl = slice(b * L, (b + 1) * L)
            ri = slice(i * L, (i + 1) * L)
            prev[sl] = r["argmax"][ri]
            if r["stop"][i] or k == N - 1:
                canvas[sl] = r["sampled"][ri]
                active[b] = False
                steps[b] = k - k_start + 1
            else:
                canvas[sl] = r["canvas"][ri]
        hp[:] = 1
        if not active.any():
            break
    assert V > 0
    return canvas, steps, history
