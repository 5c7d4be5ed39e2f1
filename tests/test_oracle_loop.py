"""Pins for the oracle's adaptive loop: stopping rule, freezing, commit."""
import numpy as np

import synth
from oracle import denoise_loop, step as S
from oracle.step import Params


def _run(B=2, L=256, d=256, V=1024, params=Params()):
    E = synth.embedder_normal(V, d, seed=1)
    y = synth.loop_targets(L, V, seed=3, B=B)
    calls = []

    def hidden(k, canvas):
        calls.append(k)
        return synth.loop_hidden(k, y, E, seed=4)

    fin, steps, hist = denoise_loop(hidden, E_bits=E, B=B, L=L, params=params)
    return E, y, fin, steps, hist, calls


def test_loop_stops_early_and_commits_sampled_tokens():
    E, y, fin, steps, hist, calls = _run()
    assert np.all(steps >= 2) and np.all(steps < 48)
    # the first step of a canvas can never stop
    assert not hist[0]["stop"].any()
    # mean entropy at the stopping step is under the threshold
    last = hist[-1]
    for i, b in enumerate(last["canvases"]):
        if last["stop"][i]:
            assert last["mean_entropy"][i] < S.STOP_ENTROPY
    # the synthetic signal points at y, so the committed canvas is y
    assert (fin == y).mean() > 0.99
    assert calls == list(range(len(hist)))


def test_loop_respects_max_steps_and_commits_at_last_step():
    p = Params(max_steps=3)
    E, y, fin, steps, hist, calls = _run(params=p)
    assert np.all(steps == 3) and len(hist) == 3
    assert not any(h["stop"].any() for h in hist)


def test_loop_entropy_falls():
    _, _, _, _, hist, _ = _run(B=1)
    me = [h["mean_entropy"][0] for h in hist]
    assert me[-1] < me[0]
    assert all(b <= a + 1e-3 for a, b in zip(me[3:], me[4:]))
