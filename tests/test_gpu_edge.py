"""Edge cases of the step on the device: degenerate logits and the largest
batch.

* All-zero embedder: every logit is 0, so the tempered distribution is
  uniform: entropy ln V, argmax the lowest index 0, and the Gumbel draw is
  decided by the noise alone (replayed bit-exactly).
* One dominant token per row: entropy ~0, the argmax and the sample are that
  token, every slot is accepted and the stop test fires on the second step.
* DG_MAX_B = 256 canvases (65,536 rows) at a small vocabulary: every canvas
  with its own step index, checked against the oracle on sampled canvases
  and structurally on all.
"""
import math

import numpy as np
import pytest

import oracle
import synth
from dg_testlib import check_replay, compare_with_oracle, oparams, run_step, seeded_inputs

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import block_canvas_denoising_b200 as dg  # noqa: E402
from block_canvas_denoising_b200 import build as dg_build  # noqa: E402

dg_build.build()
L = 256


def test_all_zero_embedder_gives_uniform_distribution():
    B, d, V = 1, 256, 4096
    h, _, canvas0 = seeded_inputs(B, d, V)
    E = np.zeros((V, d), np.uint16)
    ks = np.array([10], np.int32)
    hp = np.zeros(1, np.uint8)
    prev = np.zeros(L, np.int32)
    params = dg.Params()
    g = run_step(h, E, ks, hp, prev, canvas0, params)
    assert np.all(g["logits"] == 0.0)
    assert np.abs(g["entropy"] - math.log(V)).max() < 1e-5
    assert np.all(g["argmax"] == 0)
    # ln V per slot: the cumulative rule keeps only the lowest-entropy slot
    assert g["accept"].sum() == 1
    check_replay(g, ks, hp, prev, params)
    compare_with_oracle(g, h, E, ks, hp, prev, params)


def test_dominant_token_rows_accept_everything_and_stop():
    # h_r = 40 * E[y_r] / |E[y_r]| * sqrt(d): logit y_r is far above the rest
    B, d, V = 1, 512, 8192
    E = synth.embedder_normal(V, d, seed=1)
    y = synth.loop_targets(L, V, seed=3, B=B)
    e = synth.bf16_bits_to_f32(E[y]).astype(np.float64)
    h = synth.bf16_bits_from_f32((40.0 * e / np.linalg.norm(e, axis=1, keepdims=True) * math.sqrt(d))
                                 .astype(np.float32))
    canvas0 = synth.canvas_uniform(B, L, V, seed=0)
    params = dg.Params()
    ks = np.array([5], np.int32)
    g1 = run_step(h, E, ks, np.zeros(1, np.uint8), np.zeros(L, np.int32), canvas0, params)
    assert np.array_equal(g1["argmax"], y) and np.array_equal(g1["sampled"], y)
    assert g1["entropy"].max() < 1e-3 and g1["accept"].sum() == L
    assert g1["stop"][0] == 0                      # no previous prediction yet
    ks2 = np.array([6], np.int32)
    g2 = run_step(h, E, ks2, np.ones(1, np.uint8), g1["argmax"], g1["canvas"], params)
    assert g2["stop"][0] == 1                      # same prediction, mean entropy < 0.005
    compare_with_oracle(g2, h, E, ks2, np.ones(1, np.uint8), g1["argmax"], params)


def test_max_batch_256_canvases():
    B, d, V = dg_max_b(), 128, 512
    h, E, canvas0 = seeded_inputs(B, d, V)
    ks = synth.step_indices_uniform(B, 48, seed=5)
    hp = (np.arange(B) % 2).astype(np.uint8)
    prev = np.random.default_rng(8).integers(0, V, B * L).astype(np.int32)
    params = dg.Params()
    g = run_step(h, E, ks, hp, prev, canvas0, params)
    for b in (0, 1, 127, 255):
        compare_with_oracle(g, h, E, ks, hp, prev, params, canvases=[b])
    check_replay(g, ks, hp, prev, params, canvases=[0, 255])
    for b in range(B):
        sl = slice(b * L, (b + 1) * L)
        acc = g["accept"][sl]
        assert acc.sum() >= 1
        assert np.array_equal(g["canvas"][sl][acc == 1], g["sampled"][sl][acc == 1])
        assert np.array_equal(g["prev_argmax"][sl], g["argmax"][sl])
        assert g["stop"][b] in (0, 1)


def dg_max_b() -> int:
    import re
    import os
    hdr = open(os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "dg.h")).read()
    return int(re.search(r"#define DG_MAX_B (\d+)", hdr).group(1))
