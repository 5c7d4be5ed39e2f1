"""Pins for the oracle's adaptive loop: stopping rule, freezing, commit."""
import numpy as np
import pytest

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


# ---------------------------------------------------------------------------
# Per-canvas freeze and final commit, checked against the step function
# ---------------------------------------------------------------------------

def _two_speed_loop(params=Params(), L=256, d=256, V=1024):
    """B = 2 canvases: canvas 1's stand-in signal grows three times as fast,
    so it settles (and stops) several steps before canvas 0.  Returns the
    loop's results plus the canvas passed to every call of the hidden-state
    callback and the hidden states it returned."""
    E = synth.embedder_normal(V, d, seed=1)
    y = synth.loop_targets(L, V, seed=3, B=2)
    seen, hs = [], []

    def hidden(k, canvas):
        seen.append(np.array(canvas, copy=True))
        h = np.concatenate([synth.loop_hidden(k, y[:L], E, seed=4),
                            synth.loop_hidden(3 * k, y[L:], E, seed=5)])
        hs.append(h)
        return h

    fin, steps, hist = denoise_loop(hidden, E_bits=E, B=2, L=L, params=params)
    return E, fin, steps, hist, seen, hs


def _sampled_at(h, E, k, b, params, L=256):
    """Sampled tokens of canvas b at step k, from an independent step call
    (the draw depends only on h, k, b and the seed)."""
    from oracle import denoise_step
    r = denoise_step(h, E_bits=E, B=2, L=L, step_idx=np.full(2, k, np.int32), has_prev=np.zeros(2, np.uint8),
                     prev_argmax=np.zeros(2 * L, np.int32), params=params, canvases=[b])
    return r["sampled"]


def check_freeze_and_commit(E, fin, steps, seen, hs, params, L=256):
    """A canvas that stopped after s steps holds, from then on, exactly the
    tokens its s-th step sampled: in every later callback and at the end."""
    for b in range(2):
        sl = slice(b * L, (b + 1) * L)
        s = int(steps[b])
        committed = _sampled_at(hs[s - 1], E, s - 1, b, params)
        assert np.array_equal(fin[sl], committed), b
        for k in range(s, len(seen)):
            assert np.array_equal(seen[k][sl], committed), (b, k)


def test_loop_canvases_stop_at_different_steps_and_stay_frozen():
    p = Params()
    E, fin, steps, hist, seen, hs = _two_speed_loop(p)
    assert steps[1] < steps[0] < p.max_steps, steps
    # canvas 1 is dropped from the steps after its stop
    for h in hist[int(steps[1]):]:
        assert h["canvases"] == [0]
    # the stop fired at each canvas's last step (not the step cap)
    last1 = hist[int(steps[1]) - 1]
    assert last1["stop"][last1["canvases"].index(1)]
    check_freeze_and_commit(E, fin, steps, seen, hs, p)


def test_loop_commit_at_the_step_cap_is_the_last_sampled_canvas():
    # three steps are too few to settle: both canvases commit at k = N-1
    p = Params(max_steps=3)
    E, fin, steps, hist, seen, hs = _two_speed_loop(p)
    assert np.all(steps == 3)
    # canvas 0 never stops: it commits because the cap is reached
    assert not any(h["stop"][h["canvases"].index(0)] for h in hist)
    for b in range(2):
        sl = slice(b * 256, (b + 1) * 256)
        assert np.array_equal(fin[sl], _sampled_at(hs[2], E, 2, b, p))
        # the committed canvas is the draw, not the renoised canvas of step 2
        assert not np.array_equal(fin[sl], seen[2][sl])


def test_freeze_check_rejects_a_loop_that_keeps_updating_a_stopped_canvas():
    # planted mistake: after canvas 1 stops, later steps keep overwriting it
    p = Params()
    E, fin, steps, hist, seen, hs = _two_speed_loop(p)
    s1 = int(steps[1])
    assert len(seen) > s1
    bad = [c.copy() for c in seen]
    bad[s1][256 + 7] ^= 1
    with pytest.raises(AssertionError):
        check_freeze_and_commit(E, fin, steps, bad, hs, p)
    bad_fin = fin.copy()
    bad_fin[256 + 3] = (bad_fin[256 + 3] + 1) % 1024
    with pytest.raises(AssertionError):
        check_freeze_and_commit(E, bad_fin, steps, seen, hs, p)


def test_loop_over_a_subset_of_canvases_equals_the_full_loop_on_them():
    E = synth.embedder_normal(1024, 256, seed=1)
    y = synth.loop_targets(256, 1024, seed=3, B=3)
    hidden = lambda k, c: synth.loop_hidden(k, y, E, seed=4)   # noqa: E731
    full, steps, _ = denoise_loop(hidden, E_bits=E, B=3, L=256)
    sub, ssteps, _ = denoise_loop(hidden, E_bits=E, B=3, L=256, canvases=[2, 0])
    for b in (0, 2):
        assert np.array_equal(sub[b * 256:(b + 1) * 256], full[b * 256:(b + 1) * 256])
        assert ssteps[b] == steps[b]
    assert ssteps[1] == 0 and np.all(sub[256:512] == 0)
