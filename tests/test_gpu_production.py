"""Parity at the production sizes, in the launch configuration the bench
times: B=1, d=2816, V=262,144 at k = 0, 23, 47; batched B=8 and B=32 with a
step index and stream per canvas (sampled canvases checked against the
oracle; bit-exact replay on the device's logits of sampled canvases;
structural invariants on every canvas)."""
import numpy as np
import pytest

import oracle
import synth
from dg_testlib import check_replay, compare_with_oracle, oparams, to_dev_bf16

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import block_canvas_denoising_b200 as dg  # noqa: E402
from block_canvas_denoising_b200 import build as dg_build  # noqa: E402

dg_build.build()

D, V, L = 2816, 262144, 256


@pytest.fixture(scope="module")
def embedder():
    E_bits = synth.embedder_normal(V, D, seed=1)
    return E_bits, to_dev_bf16(E_bits)


def _run(E_dev, h_bits, ks, has_prev, prev, canvas0, params, canvases):
    """Device step with logits dumped; numpy outputs plus the logits of the
    requested canvases, keyed by canvas."""
    B = len(ks)
    R = B * L
    h = to_dev_bf16(h_bits)
    out = dict(canvas=torch.from_numpy(canvas0.copy()).cuda(),
               prev_argmax=torch.from_numpy(prev.copy()).cuda(),
               accept=torch.zeros(R, dtype=torch.uint8, device="cuda"),
               entropy=torch.zeros(R, dtype=torch.float32, device="cuda"),
               sampled=torch.zeros(R, dtype=torch.int32, device="cuda"),
               argmax=torch.zeros(R, dtype=torch.int32, device="cuda"),
               stop=torch.full((B,), -1, dtype=torch.int32, device="cuda"))
    logits = torch.empty((R, V), dtype=torch.float32, device="cuda")
    ws = dg.Workspace(B, D, V)
    dg.debug_logits(h, E_dev, ks, has_prev, out["canvas"], out["prev_argmax"], out["accept"],
                    out["entropy"], out["sampled"], out["argmax"], out["stop"], logits, ws, params)
    assert dg.device_status(ws) == 0
    g = {k: v.cpu().numpy() for k, v in out.items()}
    lg = {b: logits[b * L:(b + 1) * L].cpu().numpy() for b in canvases}
    del logits
    torch.cuda.empty_cache()
    return g, lg


def _canvas_view(g, lg, b):
    sl = slice(b * L, (b + 1) * L)
    sub = {k: v[sl] for k, v in g.items() if k != "stop"}
    sub["stop"] = g["stop"][b:b + 1]
    sub["logits"] = lg[b]
    return sub


@pytest.mark.parametrize("k", [0, 23, 47])
def test_production_single_step(embedder, k):
    E_bits, E_dev = embedder
    h_bits = synth.hidden_normal(1, L, D, seed=2)
    canvas0 = synth.canvas_uniform(1, L, V, seed=0)
    ks = np.array([k], np.int32)
    hp = np.zeros(1, np.uint8)
    prev = np.zeros(L, np.int32)
    params = dg.Params()
    g, lg = _run(E_dev, h_bits, ks, hp, prev, canvas0, params, [0])
    g["logits"] = lg[0]
    report = {}
    compare_with_oracle(g, h_bits, E_bits, ks, hp, prev, params, report=report)
    check_replay(g, ks, hp, prev, params)
    print(k, report)
    assert report["logit_rel_err"] < 1e-5


def _replay_canvas(sub, b, ks, hp, prev, params):
    rp = oracle.replay_step(sub["logits"], B=len(ks), L=L, step_idx=ks, has_prev=hp,
                            prev_argmax=prev, params=oparams(params), entropy_in=sub["entropy"],
                            canvases=[b])
    for key in ("sampled", "argmax", "accept", "canvas"):
        assert np.array_equal(rp[key], sub[key]), key
    assert rp["stop"][0] == sub["stop"][0]


def _batched(embedder, B, check_canvases, replay_canvases):
    E_bits, E_dev = embedder
    h_bits = synth.hidden_normal(B, L, D, seed=2)
    canvas0 = synth.canvas_uniform(B, L, V, seed=0)
    ks = synth.step_indices_uniform(B, 48, seed=5)
    hp = (np.arange(B) % 2).astype(np.uint8)           # half the canvases have a history
    prev = np.random.default_rng(6).integers(0, V, B * L).astype(np.int32)
    params = dg.Params()
    canv = sorted(set(check_canvases) | set(replay_canvases))
    g, lg = _run(E_dev, h_bits, ks, hp, prev, canvas0, params, canv)
    for b in check_canvases:
        sl = slice(b * L, (b + 1) * L)
        # the oracle runs this canvas alone, as canvas b of the batch
        r = oracle.denoise_step(h_bits, E_bits=E_bits, B=B, L=L, step_idx=ks, has_prev=hp,
                                prev_argmax=prev, params=oparams(params), canvases=[b])
        assert np.abs(g["entropy"][sl] - r["entropy"]).max() <= 2e-3
        bad = g["sampled"][sl] != r["sampled"]
        assert np.all(r["gumbel_margin"][bad] < 1e-3) and bad.sum() <= 1
        zb = lg[b].astype(np.float64)
        top2 = -np.partition(-zb, 1, axis=1)[:, :2]
        badm = g["argmax"][sl] != r["argmax"]
        assert np.all((top2[:, 0] - top2[:, 1])[badm] < 1e-3) and badm.sum() <= 1
        if not np.array_equal(g["accept"][sl], r["accept"]):
            assert r["order_margin"][0] < 1e-3
        if g["stop"][b] != r["stop"][0]:
            assert r["stop_margin"][0] < 1e-3
    for b in replay_canvases:
        _replay_canvas(_canvas_view(g, lg, b), b, ks, hp, prev, params)
    for b in range(B):     # structural invariants on every canvas
        sl = slice(b * L, (b + 1) * L)
        acc = g["accept"][sl]
        assert acc.sum() >= 1
        assert np.array_equal(g["canvas"][sl][acc == 1], g["sampled"][sl][acc == 1])
        assert np.all((g["sampled"][sl] >= 0) & (g["sampled"][sl] < V))
        assert g["stop"][b] in (0, 1)
        assert np.array_equal(g["prev_argmax"][sl], g["argmax"][sl])
    assert np.all(g["entropy"] >= 0)


def test_batched_b8_per_canvas_steps(embedder):
    _batched(embedder, 8, check_canvases=[0, 5], replay_canvases=[0, 3, 7])


def test_batched_b32_per_canvas_steps(embedder):
    _batched(embedder, 32, check_canvases=[31], replay_canvases=[0, 17, 31])
