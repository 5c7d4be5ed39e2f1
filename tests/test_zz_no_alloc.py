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

import synth
from dg_testlib import ENTROPY_TOL, seeded_inputs, to_dev_bf16, to_dev_fp8

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


@pytest.mark.parametrize("B,d,V,ks,hp,fp8", [
    (1, 512, 8192, [0], [0], False),
    (2, 2816, 4096, [3, 40], [1, 0], False),
    (1, 2816, 262144, [23], [1], False),
    (1, 2816, 262144, [23], [1], True),
])
def test_noalloc_matches_workspace_step_on_two_calls(B, d, V, ks, hp, fp8):
    h_bits, E_bits, canvas0 = seeded_inputs(B, d, V)
    prev = np.random.default_rng(9).integers(0, V, B * 256).astype(np.int32)
    h = to_dev_bf16(h_bits)
    if fp8:
        E, sc = to_dev_fp8(*synth.quantize_e4m3_rows(E_bits))
    else:
        E, sc = to_dev_bf16(E_bits), None
    R = B * 256
    params = dg.Params(seed=4321)

    ws = dg.Workspace(B, d, V, dg.E_FP8_E4M3 if fp8 else dg.E_BF16)
    ref = _buffers(R, B, canvas0, prev)
    dg.denoise_step(h, E, ks, hp, *_args(ref), ws, params, e_scale=sc)
    torch.cuda.synchronize()
    assert dg.device_status(ws) == 0
    ref = {k: v.cpu().numpy() for k, v in ref.items()}

    for call in range(2):
        out = _buffers(R, B, canvas0, prev)
        dg.denoise_step_noalloc(h, E, ks, hp, *_args(out), params, e_scale=sc)
        torch.cuda.synchronize()
        assert dg.noalloc_status() == 0
        out = {k: v.cpu().numpy() for k, v in out.items()}
        for key in ("canvas", "prev_argmax", "accept", "sampled", "argmax", "stop"):
            assert np.array_equal(out[key], ref[key]), (call, key)
        assert np.abs(out["entropy"].astype(np.float64) - ref["entropy"]).max() <= ENTROPY_TOL, call


def _refused(B, e_dtype):
    L = dg.lib()
    shp = dg._Shape(B, 256, 2816, 262144, e_dtype)
    prm = dg.Params().c()
    ks = np.zeros(B, np.int32)
    hpv = np.zeros(B, np.uint8)
    fake = ctypes.c_void_p(256)
    scale = fake if e_dtype == dg.E_FP8_E4M3 else None
    return L.dg_denoise_step_noalloc(ctypes.byref(shp), ctypes.byref(prm), fake, fake, scale,
                                     ks.ctypes.data_as(ctypes.c_void_p), hpv.ctypes.data_as(ctypes.c_void_p),
                                     None, fake, fake, fake, fake, fake, fake, fake, None)


@pytest.mark.parametrize("B,e_dtype,fits", [(32, dg.E_BF16, False), (19, dg.E_BF16, False), (18, dg.E_BF16, True),
                                            (3, dg.E_FP8_E4M3, False), (2, dg.E_FP8_E4M3, True)])
def test_noalloc_refuses_exactly_the_shapes_beyond_its_scratch(B, e_dtype, fits):
    # over the 262,144-token vocabulary on a 148-SM B200: B = 19 and 32 bf16
    # canvases need about 8.7 and 14.7 MB of scratch and B = 3 with the FP8
    # embedder about 9.8 MB (its scratch also holds h's two E4M3 terms), while
    # B = 18 bf16 (about 8.3 MB) and B = 2 FP8 fit the 8 MiB array
    need = dg.workspace_size(B, 2816, 262144, e_dtype)
    assert (need <= 8 * 1024 * 1024) == fits, need
    if fits:
        return          # a fitting shape would run: not called with placeholder pointers
    # refused before anything runs, so the placeholder pointers are never used
    code = _refused(B, e_dtype)
    assert code == 3    # DG_ERR_WORKSPACE
    msg = dg.lib().dg_last_error_message().decode()
    assert "scratch" in msg and "bytes" in msg


def test_noalloc_reports_a_latched_fault_then_runs_clean():
    # the bounded-wait self test latches a timeout in the shared array (it
    # gives up after 2 ms, nothing hangs); the status call reports it once
    # and clears it, and the next step runs with a clean latch
    assert dg.noalloc_selftest_bounded_wait(2_000_000) == 6   # DG_ERR_TIMEOUT
    assert dg.noalloc_status() == 0
    B, d, V = 1, 512, 8192
    h_bits, E_bits, canvas0 = seeded_inputs(B, d, V)
    out = _buffers(256, B, canvas0, np.zeros(256, np.int32))
    dg.denoise_step_noalloc(to_dev_bf16(h_bits), to_dev_bf16(E_bits), [0], [0], *_args(out))
    assert dg.noalloc_status() == 0
    assert int(out["accept"].sum()) >= 1
