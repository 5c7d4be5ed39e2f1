"""GPU parity of the fused step against the CPU oracle (through the C ABI).

Shapes span one to many tiles with ragged splits: d from one K stage (64)
to the production 2816, V from one vocabulary tile (256) to 262,144, B up to
8 with per-canvas step indices.  Every case checks the stated tolerances and
the bit-exact replay of the sampler on the device's own logits.
"""
import numpy as np
import pytest

import synth
from dg_testlib import check_replay, compare_with_oracle, run_step, seeded_inputs

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import block_canvas_denoising_b200 as dg  # noqa: E402
from block_canvas_denoising_b200 import build as dg_build  # noqa: E402

dg_build.build()


def _case(B, d, V, ks, has_prev=None, params=None, seeds=(2, 1, 0), prev=None):
    params = params or dg.Params()
    h, E, canvas0 = seeded_inputs(B, d, V, h_seed=seeds[0], e_seed=seeds[1], canvas_seed=seeds[2])
    has_prev = np.zeros(B, np.uint8) if has_prev is None else np.asarray(has_prev, np.uint8)
    prev = np.zeros(B * 256, np.int32) if prev is None else prev
    ks = np.asarray(ks, np.int32)
    g = run_step(h, E, ks, has_prev, prev, canvas0, params)
    return h, E, ks, has_prev, prev, params, g


def test_tiny_config_parity_and_replay():
    # B=1, L=256, d=512, V=8192, k=0 (tau 0.8), canvas seed 0, Philox seed 1234
    h, E, ks, hp, prev, params, g = _case(1, 512, 8192, [0])
    report = {}
    compare_with_oracle(g, h, E, ks, hp, prev, params, report=report)
    check_replay(g, ks, hp, prev, params)
    assert report["logit_rel_err"] < 1e-5
    assert g["stop"][0] == 0


@pytest.mark.parametrize("B,d,V,ks", [
    (1, 64, 256, [5]),            # one K stage, one vocabulary tile
    (2, 192, 768, [0, 47]),       # KB < stages, 3 tiles (ragged split)
    (3, 320, 2304, [10, 20, 30]), # 9 tiles, three canvases
    (1, 2816, 4096, [23]),        # production d, 16 tiles
    (2, 1024, 65536, [1, 46]),    # many tiles per CTA
])
def test_small_shapes_parity_and_replay(B, d, V, ks):
    h, E, ks, hp, prev, params, g = _case(B, d, V, ks)
    compare_with_oracle(g, h, E, ks, hp, prev, params)
    check_replay(g, ks, hp, prev, params)


def test_deterministic_repeat():
    h, E, canvas0 = seeded_inputs(2, 512, 8192)
    ks = np.array([3, 9], np.int32)
    hp = np.zeros(2, np.uint8)
    prev = np.zeros(512, np.int32)
    a = run_step(h, E, ks, hp, prev, canvas0, dg.Params())
    b = run_step(h, E, ks, hp, prev, canvas0, dg.Params())
    for k in ("canvas", "accept", "entropy", "sampled", "argmax", "stop", "logits"):
        assert np.array_equal(a[k], b[k]), k


def test_stop_fires_only_with_previous_prediction():
    # peaked logits (h aligned with E rows) -> near-zero entropy
    B, d, V = 1, 256, 2048
    E = synth.embedder_normal(V, d, seed=1)
    y = synth.loop_targets(256, V, seed=3)
    h = synth.loop_hidden(40, y, E, seed=4)
    params = dg.Params()
    ks = np.array([47], np.int32)
    canvas0 = synth.canvas_uniform(1, 256, V)
    g0 = run_step(h, E, ks, np.zeros(1, np.uint8), np.zeros(256, np.int32), canvas0, params)
    assert g0["entropy"].mean() < params.stop_entropy
    assert g0["stop"][0] == 0                         # first step never stops
    g1 = run_step(h, E, ks, np.ones(1, np.uint8), g0["argmax"], canvas0, params)
    assert g1["stop"][0] == 1
    other = g0["argmax"].copy()
    other[5] = (other[5] + 1) % V
    g2 = run_step(h, E, ks, np.ones(1, np.uint8), other, canvas0, params)
    assert g2["stop"][0] == 0
    compare_with_oracle(g1, h, E, ks, np.ones(1, np.uint8), g0["argmax"], params)


@pytest.mark.parametrize("B,active", [(2, [1, 0]), (4, [0, 1, 0, 1]), (3, [0, 0, 1])])
def test_frozen_canvases_untouched_and_active_ones_exact(B, active):
    # frozen canvases cost no work and keep every output; the updated ones
    # equal the same canvases of a step that updates every canvas
    h, E, canvas0 = seeded_inputs(B, 256, 1024)
    ks = np.array([4 + b for b in range(B)], np.int32)
    prev = np.full(B * 256, 7, np.int32)
    hp = np.zeros(B, np.uint8)
    g = run_step(h, E, ks, hp, prev, canvas0, dg.Params(), active=active, debug=False)
    full = run_step(h, E, ks, hp, prev, canvas0, dg.Params(), debug=False)
    for b in range(B):
        sl = slice(b * 256, (b + 1) * 256)
        if active[b]:
            for key in ("canvas", "prev_argmax", "accept", "entropy", "sampled", "argmax"):
                assert np.array_equal(g[key][sl], full[key][sl]), (b, key)
            assert g["stop"][b] == full["stop"][b]
        else:
            assert np.array_equal(g["canvas"][sl], canvas0[sl])
            assert np.all(g["prev_argmax"][sl] == 7)
            assert np.all(g["entropy"][sl] == 0) and np.all(g["sampled"][sl] == 0)
            assert np.all(g["argmax"][sl] == 0) and np.all(g["accept"][sl] == 0)
            assert g["stop"][b] == -1


def test_every_canvas_frozen_launches_nothing():
    h, E, canvas0 = seeded_inputs(2, 256, 1024)
    g = run_step(h, E, [3, 3], np.zeros(2, np.uint8), np.zeros(512, np.int32), canvas0, dg.Params(),
                 active=[0, 0], debug=False)
    assert np.array_equal(g["canvas"], canvas0) and np.all(g["stop"] == -1)


def test_bounded_wait_selftest_then_step_still_works():
    ws = dg.Workspace(1, 64, 256)
    assert dg.selftest_bounded_wait(2_000_000, ws) == 6   # timed out as designed
    assert dg.device_status(ws) == 0                       # latch cleared
    h, E, ks, hp, prev, params, g = _case(1, 64, 256, [0])
    compare_with_oracle(g, h, E, ks, hp, prev, params)
