"""dg_denoise_step_noalloc against dg_denoise_step.

The allocation-free entry point serves callers that cannot allocate device
memory where they run a step (a serving runtime that owns all GPU memory, or
code that must not call the CUDA allocator there): its scratch is a fixed
array inside the library instead of a caller workspace.  On the same inputs
it must give the same step as the workspace entry point -- integer outputs
exactly, entropies within the parity tolerance -- on two calls in a row
(the second call reuses the array the first one left behind).  Shapes whose
scratch does not fit are refused before anything runs.

This file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest

from dg_testlib import ENTROPY_TOL, seeded_inputs, to_dev_bf16

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import block_canvas_denoising_b200 as dg  # noqa: E402
from block_canvas_denoising_b200 import build as dg_build  # noqa: E402

dg_build.build()


def _buffers(R, B, canvas0, prev):
    return dict(canvas=torch.from_numpy(canvas0.copy()).cuda(),
                prev_argmax=torch.from_numpy(prev.copy()).cuda(),
                accept=torch.zeros(R, dtype=torch.uint8, device="cuda"),
                entropy=torch.zeros(R, dtype=torch.float32, device="cuda"),
                sampled=torch.zeros(R, dtype=torch.int32, device="cuda"),
                argmax=torch.zeros(R, dtype=torch.int32, device="cuda"),
                stop=torch.full((B,), -1, dtype=torch.int32, device="cuda"))


def _args(o):
    return (o["canvas"], o["prev_argmax"], o["accept"], o["entropy"], o["sampled"], o["argmax"], o["stop"])


@pytest.mark.parametrize("B,d,V,ks,hp", [
    (1, 512, 8192, [0], [0]),
    (2, 2816, 4096, [3, 40], [1, 0]),
    (1, 2816, 262144, [23], [1]),
])
def test_noalloc_matches_workspace_step_on_two_calls(B, d, V, ks, hp):
    h_bits, E_bits, canvas0 = seeded_inputs(B, d, V)
    prev = np.random.default_rng(9).integers(0, V, B * 256).astype(np.int32)
    h = to_dev_bf16(h_bits)
    E = to_dev_bf16(E_bits)
    R = B * 256
    params = dg.Params(seed=4321)

    ws = dg.Workspace(B, d, V)
    ref = _buffers(R, B, canvas0, prev)
    dg.denoise_step(h, E, ks, hp, *_args(ref), ws, params)
    torch.cuda.synchronize()
    assert dg.device_status(ws) == 0
    ref = {k: v.cpu().numpy() for k, v in ref.items()}

    for call in range(2):
        out = _buffers(R, B, canvas0, prev)
        dg.denoise_step_noalloc(h, E, ks, hp, *_args(out), params)
        torch.cuda.synchronize()
        out = {k: v.cpu().numpy() for k, v in out.items()}
        for key in ("canvas", "prev_argmax", "accept", "sampled", "argmax", "stop"):
            assert np.array_equal(out[key], ref[key]), (call, key)
        assert np.abs(out["entropy"].astype(np.float64) - ref["entropy"]).max() <= ENTROPY_TOL, call


def test_noalloc_refuses_shapes_beyond_its_scratch():
    # B = 8 canvases over the 262,144-token vocabulary need about 29 MiB of
    # scratch: refused up front, so no tensor is touched (the fake pointers
    # are never dereferenced)
    L = dg.lib()
    shp = dg._Shape(8, 256, 2816, 262144, 0)
    prm = dg.Params().c()
    ks = np.zeros(8, np.int32)
    hpv = np.zeros(8, np.uint8)
    fake = ctypes.c_void_p(256)
    code = L.dg_denoise_step_noalloc(ctypes.byref(shp), ctypes.byref(prm), fake, fake, None,
                                     ks.ctypes.data_as(ctypes.c_void_p), hpv.ctypes.data_as(ctypes.c_void_p),
                                     None, fake, fake, fake, fake, fake, fake, fake, None)
    assert code == 3    # DG_ERR_WORKSPACE
    msg = L.dg_last_error_message().decode()
    assert "scratch" in msg and "bytes" in msg
