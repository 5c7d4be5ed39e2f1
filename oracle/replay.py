"""Replay of the sampler on given float32 logits.

Fed the raw float32 logits z of a device step, this recomputes the draw with
the float32 key of ``oracle.flog`` (``fl32(fl32(z * inv_tau) + g32(u))``), the
argmax prediction of z, and -- from the entropies (either recomputed here in
float64 from z, or the device's own) -- the selection, renoise and stop of
``oracle.step``.  Tokens and argmax are then a pure function of the logits,
so they must agree bit for bit with the device.

TEST INFRASTRUCTURE: part of the CPU oracle (see ``oracle/__init__``).
"""
from __future__ import annotations

import numpy as np

from .flog import gumbel_f32, uniform_f32
from .step import (Params, argmax_lowest, counter_step, entropy, gumbel_words, inv_tau_f32,
                   renoise_tokens, select, stop_flag)


def key_f32(z32: np.ndarray, inv_tau32: np.float32, words: np.ndarray) -> np.ndarray:
    """The float32 Gumbel key of every logit."""
    x32 = np.asarray(z32, dtype=np.float32) * np.float32(inv_tau32)
    return x32 + gumbel_f32(uniform_f32(words))


def replay_step(z32, *, B: int, L: int, step_idx, has_prev, prev_argmax,
                params: Params = Params(), entropy_in=None, canvases=None,
                slot_chunk: int = 32):
    """Replay canvases ``canvases`` of a step from float32 logits [rows, V].

    ``z32`` holds the rows of the chosen canvases in order (L rows each).
    If ``entropy_in`` (float32 per row, same rows) is given, selection and
    stop use it; otherwise the entropy is recomputed in float64 from
    ``z32 * inv_tau32``.
    """
    z32 = np.asarray(z32, dtype=np.float32)
    V = z32.shape[1]
    canvases = list(range(B)) if canvases is None else [int(c) for c in canvases]
    res = {k: [] for k in ("entropy", "sampled", "argmax", "accept", "canvas")}
    stops, margins = [], []
    for i, b in enumerate(canvases):
        k = int(step_idx[b])
        it = inv_tau_f32(k, params.tau0, params.tau1, params.max_steps)
        zc = z32[i * L:(i + 1) * L]
        samp = np.empty(L, dtype=np.int32)
        H = np.empty(L)
        for s0 in range(0, L, slot_chunk):
            s1 = min(L, s0 + slot_chunk)
            w = gumbel_words(np.arange(s0, s1), b, counter_step(k, params.block), V, params.seed)
            samp[s0:s1] = np.argmax(key_f32(zc[s0:s1], it, w), axis=1)
            H[s0:s1] = entropy(zc[s0:s1].astype(np.float64) * np.float64(it))
        if entropy_in is not None:
            H = np.asarray(entropy_in[i * L:(i + 1) * L], dtype=np.float64)
        amax = argmax_lowest(zc)
        acc, _, om = select(H, params.entropy_bound, params.selection_rule, params.top_k)
        noise = renoise_tokens(b, counter_step(k, params.block), L, V, params.seed)
        canvas = np.where(acc == 1, samp, noise).astype(np.int32)
        st, _ = stop_flag(H, amax, prev_argmax[b * L:(b + 1) * L], bool(has_prev[b]),
                          params.stop_entropy)
        for key, val in (("entropy", H), ("sampled", samp), ("argmax", amax),
                         ("accept", acc), ("canvas", canvas)):
            res[key].append(val)
        stops.append(st)
        margins.append(om)
    out = {key: np.concatenate(v) for key, v in res.items()}
    out["stop"] = np.array(stops, dtype=np.int32)
    out["order_margin"] = np.array(margins)
    return out
