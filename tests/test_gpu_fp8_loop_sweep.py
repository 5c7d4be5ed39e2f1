"""The FP8-E4M3 embedder through the adaptive loop at the production shape.

E quantised per vocabulary row to E4M3 codes with a float32 scale
(absmax / 448), h bf16; d = 2816, V = 262,144, L = 256 and B in {1, 4, 16,
32} canvases, run through ``dg_denoise_loop`` on the loop's synthetic
stand-in hidden states (signal growing with k, targets seed 3, noise seed 4 +
k).  For sampled canvases the stop step and the committed canvas must equal
the oracle's loop (which dequantises E to float64), unless the oracle's stop
decision at the earlier step was a near-tie; every canvas must stop early
and commit its targets.
"""
import numpy as np
import pytest

import oracle
import synth
from dg_testlib import oparams, to_dev_bf16, to_dev_fp8

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
    q, s = synth.quantize_e4m3_rows(E_bits)
    Eq, sc = to_dev_fp8(q, s)
    return E_bits, q, s, Eq, sc


@pytest.mark.parametrize("B,check", [(1, [0]), (4, [3]), (16, [0, 9]), (32, [31])])
def test_fp8_loop_sweep_production_shape(embedder, B, check):
    E_bits, q, s, Eq, sc = embedder
    R = B * L
    y = synth.loop_targets(L, V, seed=3, B=B)
    params = dg.Params()
    h_buf = torch.empty((R, D), dtype=torch.bfloat16, device="cuda")
    canvas0 = synth.canvas_uniform(B, L, V, seed=0)
    canvas = torch.from_numpy(canvas0.copy()).cuda()
    prev = torch.zeros(R, dtype=torch.int32, device="cuda")
    hp = np.zeros(B, np.uint8)
    outs = [torch.zeros(R, dtype=torch.uint8, device="cuda"), torch.zeros(R, dtype=torch.float32, device="cuda"),
            torch.zeros(R, dtype=torch.int32, device="cuda"), torch.zeros(R, dtype=torch.int32, device="cuda"),
            torch.zeros(B, dtype=torch.int32, device="cuda")]
    ws = dg.Workspace(B, D, V, dg.E_FP8_E4M3)

    def hidden(k, canvas_t, h_t):
        h_t.copy_(to_dev_bf16(synth.loop_hidden(k, y, E_bits, seed=4)))

    steps = dg.denoise_loop(Eq, hidden, h_buf, canvas, prev, hp, *outs, ws, params, e_scale=sc)
    torch.cuda.synchronize()
    got = canvas.cpu().numpy()
    print("B", B, "steps", np.bincount(steps))
    # every canvas stops early and commits its targets
    assert np.all((steps >= 2) & (steps < 48)), steps
    assert (got == y).mean() > 0.99

    fin, osteps, hist = oracle.denoise_loop(lambda k, c: synth.loop_hidden(k, y, E_bits, seed=4), q=q, s=s,
                                            B=B, L=L, params=oparams(params), canvas=canvas0, canvases=check)
    for b in check:
        sl = slice(b * L, (b + 1) * L)
        if steps[b] != osteps[b]:
            kk = int(min(steps[b], osteps[b])) - 1
            i = hist[kk]["canvases"].index(b)
            assert abs(float(hist[kk]["mean_entropy"][i]) - params.stop_entropy) < 1e-3, (b, steps[b], osteps[b])
        else:
            assert (got[sl] != fin[sl]).sum() <= 1, b
