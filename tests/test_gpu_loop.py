"""The adaptive loop through the C ABI (dg_denoise_loop) against the oracle
loop, on the synthetic hidden-state stand-in: same stopping step, same
committed canvas; resume from an interrupted state; callback failure."""
import numpy as np
import pytest

import oracle
import synth
from dg_testlib import oparams, to_dev_bf16

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import block_canvas_denoising_b200 as dg  # noqa: E402
from block_canvas_denoising_b200 import build as dg_build  # noqa: E402

dg_build.build()
L = 256


class LoopState:
    """Device loop state: canvas, previous prediction, has-previous flags."""

    def __init__(self, B, V):
        self.canvas = torch.from_numpy(synth.canvas_uniform(B, L, V, seed=0)).cuda()
        self.prev = torch.zeros(B * L, dtype=torch.int32, device="cuda")
        self.has_prev = np.zeros(B, np.uint8)


def _gpu_loop(E_bits, y, B, params, k_start=0, state=None, fail_at=None):
    d = E_bits.shape[1]
    V = E_bits.shape[0]
    R = B * L
    E = to_dev_bf16(E_bits)
    h_buf = torch.empty((R, d), dtype=torch.bfloat16, device="cuda")
    st = state if state is not None else LoopState(B, V)
    outs = dict(accept=torch.zeros(R, dtype=torch.uint8, device="cuda"),
                entropy=torch.zeros(R, dtype=torch.float32, device="cuda"),
                sampled=torch.zeros(R, dtype=torch.int32, device="cuda"),
                argmax=torch.zeros(R, dtype=torch.int32, device="cuda"),
                stop=torch.zeros(B, dtype=torch.int32, device="cuda"))
    ws = dg.Workspace(B, d, V)
    seen = []

    def hidden(k, canvas_t, h_t):
        if fail_at is not None and k == fail_at:
            raise RuntimeError("planted callback failure")
        seen.append(k)
        h_t.copy_(to_dev_bf16(synth.loop_hidden(k, y, E_bits, seed=4)))

    steps = dg.denoise_loop(E, hidden, h_buf, st.canvas, st.prev, st.has_prev, outs["accept"],
                            outs["entropy"], outs["sampled"], outs["argmax"], outs["stop"], ws,
                            params, k_start=k_start)
    torch.cuda.synchronize()
    return st.canvas.cpu().numpy(), steps, seen


def _agree(canvas, steps, fin, osteps, hist, params):
    """Same stopping step and committed canvas, unless the oracle's stop
    decision at the earlier of the two steps was a near-tie (< 1e-3)."""
    for b in range(len(steps)):
        sl = slice(b * L, (b + 1) * L)
        if steps[b] != osteps[b]:
            k = int(min(steps[b], osteps[b])) - 1
            h = hist[k]
            i = h["canvases"].index(b)
            assert abs(float(h["mean_entropy"][i]) - params.stop_entropy) < 1e-3
        else:
            assert (canvas[sl] != fin[sl]).sum() <= 1


def _oracle_loop(E_bits, y, B, params, k_start=0):
    V = E_bits.shape[0]
    kw = {"canvas": synth.canvas_uniform(B, L, V, seed=0)}
    return oracle.denoise_loop(lambda k, c: synth.loop_hidden(k, y, E_bits, seed=4), E_bits=E_bits,
                               B=B, L=L, params=oparams(params), k_start=k_start, **kw)


@pytest.mark.parametrize("B,d,V", [(1, 256, 1024), (3, 512, 8192)])
def test_loop_matches_oracle(B, d, V):
    E_bits = synth.embedder_normal(V, d, seed=1)
    y = synth.loop_targets(L, V, seed=3, B=B)
    params = dg.Params()
    canvas, steps, seen = _gpu_loop(E_bits, y, B, params)
    fin, osteps, hist = _oracle_loop(E_bits, y, B, params)
    _agree(canvas, steps, fin, osteps, hist, params)
    assert seen == list(range(int(steps.max())))


def test_loop_resume_equals_uninterrupted():
    B, d, V = 2, 256, 1024
    E_bits = synth.embedder_normal(V, d, seed=1)
    y = synth.loop_targets(L, V, seed=3, B=B)
    params = dg.Params()
    full_canvas, full_steps, _ = _gpu_loop(E_bits, y, B, params)
    assert full_steps.min() > 3
    # interrupted: the callback fails at k = 3, leaving the state after step 2
    st = LoopState(B, V)
    with pytest.raises(dg.DGError) as ei:
        _gpu_loop(E_bits, y, B, params, state=st, fail_at=3)
    assert ei.value.code == 7          # DG_ERR_CALLBACK
    assert np.all(st.has_prev == 1)
    canvas, steps, seen = _gpu_loop(E_bits, y, B, params, k_start=3, state=st)
    assert seen[0] == 3
    assert np.array_equal(canvas, full_canvas)
    assert np.array_equal(steps + 3, full_steps)


def test_loop_production_shape():
    d, V = 2816, 262144
    E_bits = synth.embedder_normal(V, d, seed=1)
    y = synth.loop_targets(L, V, seed=3)
    params = dg.Params()
    canvas, steps, _ = _gpu_loop(E_bits, y, 1, params)
    fin, osteps, hist = _oracle_loop(E_bits, y, 1, params)
    print("steps", steps, osteps, [(h["k"], float(h["mean_entropy"][0]), int(h["n_accept"][0])) for h in hist])
    _agree(canvas, steps, fin, osteps, hist, params)
    assert (canvas == y).mean() > 0.99
