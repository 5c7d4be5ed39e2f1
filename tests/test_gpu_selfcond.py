"""The self-conditioning signal s = softmax(z / tau) E through the C ABI
against the float64 oracle (``oracle.selfcond.expected_embedding``).

The device rounds the probabilities to bf16 twice (block-scaled in the head,
then normalised), so each weight carries a relative error of at most
2 * 2^-9 = 2^-8, and the signal's error is bounded elementwise by
2^-8 * sum_v p_v |E[v, c]| (the oracle's ``abs_values`` scale) plus the
float32 sums (slack 2^-12 of the same scale).  The step that carries the
signal must give dg_denoise_step's results bit for bit.
"""
import numpy as np
import pytest

import synth
from dg_testlib import run_step, seeded_inputs, to_dev_bf16, to_dev_fp8

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import block_canvas_denoising_b200 as dg  # noqa: E402
from block_canvas_denoising_b200 import build as dg_build  # noqa: E402
from oracle import selfcond  # noqa: E402

dg_build.build()
L = 256
BOUND = 2.0 ** -8 + 2.0 ** -12


def _selfcond_step(h_bits, E_bits, ks, hp, prev, canvas0, params, q=None, s=None):
    B = len(ks)
    R, d = h_bits.shape
    V = E_bits.shape[0] if q is None else q.shape[0]
    h = to_dev_bf16(h_bits)
    if q is None:
        E, sc, e_dtype = to_dev_bf16(E_bits), None, dg.E_BF16
    else:
        (E, sc), e_dtype = to_dev_fp8(q, s), dg.E_FP8_E4M3
    Et = torch.empty((d, V), dtype=torch.bfloat16, device="cuda")
    dg.embedder_transpose(E, Et, e_fp8=q is not None)
    out = dict(canvas=torch.from_numpy(np.asarray(canvas0, np.int32).copy()).cuda(),
               prev_argmax=torch.from_numpy(np.asarray(prev, np.int32).copy()).cuda(),
               accept=torch.zeros(R, dtype=torch.uint8, device="cuda"),
               entropy=torch.zeros(R, dtype=torch.float32, device="cuda"),
               sampled=torch.zeros(R, dtype=torch.int32, device="cuda"),
               argmax=torch.zeros(R, dtype=torch.int32, device="cuda"),
               stop=torch.full((B,), -1, dtype=torch.int32, device="cuda"))
    signal = torch.full((R, d), float("nan"), dtype=torch.float32, device="cuda")
    ws = dg.Workspace(B, d, V, e_dtype, selfcond=True)
    dg.denoise_step_selfcond(h, E, Et, ks, hp, out["canvas"], out["prev_argmax"], out["accept"], out["entropy"],
                             out["sampled"], out["argmax"], out["stop"], signal, ws, params, e_scale=sc)
    assert dg.device_status(ws) == 0
    torch.cuda.synchronize()
    res = {k: v.cpu().numpy() for k, v in out.items()}
    res["signal"] = signal.cpu().numpy()
    # the transpose itself: E_t[c, v] = E[v, c]
    if q is None:
        et = Et.view(torch.int16).cpu().numpy().view(np.uint16)
        assert np.array_equal(et, np.asarray(E_bits).T)
    return res


def _check(res, h_bits, E_bits, ks, hp, prev, canvas0, params, q=None, s=None, rows=None):
    B = len(ks)
    emb = dict(E_bits=E_bits) if q is None else dict(q=q, s=s)
    # the same step as dg_denoise_step, bit for bit
    ref = run_step(h_bits, E_bits if q is None else q, ks, hp, prev, canvas0, params, debug=False, e_scale=s)
    for key in ("canvas", "prev_argmax", "accept", "sampled", "argmax", "stop"):
        assert np.array_equal(res[key], ref[key]), key
    assert np.array_equal(res["entropy"].view(np.uint32), ref["entropy"].view(np.uint32))
    worst = 0.0
    for b in range(B):
        sl = slice(b * L, (b + 1) * L) if rows is None else rows
        hb = h_bits[sl]
        want = selfcond.expected_embedding(hb, **emb, k=int(ks[b]))
        scale = selfcond.expected_embedding(hb, **emb, k=int(ks[b]), abs_values=True)
        got = res["signal"][sl].astype(np.float64)
        assert np.all(np.isfinite(got))
        err = np.abs(got - want)
        assert np.all(err <= BOUND * scale + 1e-12), float((err / np.maximum(scale, 1e-30)).max())
        worst = max(worst, float((err / np.maximum(scale, 1e-30)).max()))
        if rows is not None:
            break
    return worst


@pytest.mark.parametrize("B,d,V,ks", [(1, 256, 4096, [0]), (2, 512, 8192, [3, 40]), (1, 2816, 16384, [23])])
def test_selfcond_signal_matches_oracle(B, d, V, ks):
    h, E, canvas0 = seeded_inputs(B, d, V)
    ks = np.array(ks, np.int32)
    hp = np.zeros(B, np.uint8)
    prev = np.zeros(B * L, np.int32)
    params = dg.Params()
    res = _selfcond_step(h, E, ks, hp, prev, canvas0, params)
    worst = _check(res, h, E, ks, hp, prev, canvas0, params)
    print("worst relative error", worst)


def test_selfcond_low_entropy_and_uniform_rows():
    # confident slots (the loop stand-in at step 5): the signal is close to
    # E[y]; h = 0 rows: uniform distribution, the signal is E's mean row
    B, d, V = 2, 512, 8192
    E = synth.embedder_normal(V, d, seed=1)
    y = synth.loop_targets(L, V, seed=3, B=B)
    h = synth.loop_hidden(5, y, E, seed=4)
    h[L:L + 64] = 0
    ks = np.array([5, 5], np.int32)
    hp = np.ones(B, np.uint8)
    prev = np.zeros(B * L, np.int32)
    canvas0 = synth.canvas_uniform(B, L, V, seed=0)
    res = _selfcond_step(h, E, ks, hp, prev, canvas0, dg.Params())
    _check(res, h, E, ks, hp, prev, canvas0, dg.Params())
    mean_row = synth.bf16_bits_to_f32(E).astype(np.float64).mean(axis=0)
    assert np.abs(res["signal"][L:L + 64] - mean_row[None, :]).max() < 2.0 ** -8 * np.abs(mean_row).max() + 1e-4


def test_selfcond_fp8_embedder():
    B, d, V = 1, 512, 8192
    h, E, canvas0 = seeded_inputs(B, d, V)
    q, s = synth.quantize_e4m3_rows(E)
    ks = np.array([10], np.int32)
    hp = np.zeros(B, np.uint8)
    prev = np.zeros(B * L, np.int32)
    res = _selfcond_step(h, E, ks, hp, prev, canvas0, dg.Params(), q=q, s=s)
    _check(res, h, E, ks, hp, prev, canvas0, dg.Params(), q=q, s=s)


def test_selfcond_production_shape():
    # the bench workload: B = 1, d = 2816, V = 262,144, k = 0; every row
    d, V = 2816, 262144
    h, E, canvas0 = seeded_inputs(1, d, V)
    ks = np.array([0], np.int32)
    hp = np.zeros(1, np.uint8)
    prev = np.zeros(L, np.int32)
    res = _selfcond_step(h, E, ks, hp, prev, canvas0, dg.Params())
    worst = _check(res, h, E, ks, hp, prev, canvas0, dg.Params())
    print("worst relative error", worst)
