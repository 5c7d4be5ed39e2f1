"""GPU checks of the two Gumbel transforms the fused sampler uses.

* The specified float32 transform g32 = -L(-L(u)) computed on the device is
  bit-identical to the oracle's for every one of the 2^23 possible u.
* The screening approximation (hardware lg2 based) stays within the error
  bound the kernel assumes, over the same exhaustive set of inputs.
"""
import numpy as np
import pytest

from oracle import flog

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import block_canvas_denoising_b200 as dg  # noqa: E402
from block_canvas_denoising_b200 import build as dg_build  # noqa: E402

dg_build.build()

KERNEL_BOUND = 1.0e-5   # kGumbelApproxErr in the kernel
LN2_F32 = float(np.float32(0.693147182464599609375))
C0_F32 = float(np.float32(0.36651292058166432))   # -ln(ln 2), kGumbelC0


def _all_levels():
    # u depends on r >> 9 only: one word per level, plus random low bits
    levels = np.arange(1 << 23, dtype=np.uint64)
    low = np.random.default_rng(0).integers(0, 512, size=1 << 23, dtype=np.uint64)
    return ((levels << np.uint64(9)) | low).astype(np.uint32)


def test_exact_transform_bit_identical_for_every_u():
    w = _all_levels()
    wt = torch.from_numpy(w.view(np.int32)).cuda()
    g, _ = dg.debug_gumbel(wt)
    g = g.cpu().numpy()
    ref = flog.gumbel_f32(flog.uniform_f32(w))
    assert np.array_equal(g.view(np.uint32), ref.view(np.uint32))


def test_approximation_within_kernel_bound_for_every_u():
    w = _all_levels()
    wt = torch.from_numpy(w.view(np.int32)).cuda()
    g, a = dg.debug_gumbel(wt)
    g = g.cpu().numpy().astype(np.float64)
    approx = C0_F32 - LN2_F32 * a.cpu().numpy().astype(np.float64)
    err = np.abs(approx - g).max()
    print("max |g_approx - g32| =", err)
    assert err < 0.5 * KERNEL_BOUND, err
