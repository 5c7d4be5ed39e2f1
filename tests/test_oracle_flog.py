"""Pins for the float32 log and Gumbel transform that define the sampler key.

The float32 definition must be an accurate natural log (checked against the
C library's double-precision log over sweeps and edge cases) and its Gumbel
transform an accurate -ln(-ln u) (checked against float64).
"""
import math

import numpy as np

from oracle import flog


def _ulp32(v):
    return np.spacing(np.abs(v).astype(np.float32)).astype(np.float64)


def _check_log(y, max_ulp=2.5):
    y = np.asarray(y, dtype=np.float32)
    got = flog.log_f32(y).astype(np.float64)
    ref = np.log(y.astype(np.float64))
    err = np.abs(got - ref)
    # relative to the result's ulp, with an absolute floor near ln = 0
    tol = max_ulp * np.maximum(_ulp32(ref), 2.0 ** -49)
    bad = err > tol
    assert not bad.any(), (y[bad][:5], got[bad][:5], ref[bad][:5])


def test_log_random_sweep():
    g = np.random.default_rng(0)
    _check_log(g.uniform(1e-7, 1.0, 200000))
    _check_log(g.uniform(1.0, 40.0, 200000))
    _check_log(np.exp(g.uniform(-80, 80, 200000)))


def test_log_edges():
    pw = np.ldexp(np.float32(1.0), np.arange(-126, 128)).astype(np.float32)
    _check_log(pw)
    s2 = np.float32(math.sqrt(2.0))
    around = np.array([np.nextafter(s2, np.float32(0)), s2, np.nextafter(s2, np.float32(2))],
                      dtype=np.float32)
    _check_log(around)
    _check_log(around * np.float32(0.25))
    near1 = (np.float32(1.0) + np.arange(-4096, 4097, dtype=np.float32) * np.float32(2.0 ** -24))
    _check_log(near1[near1 > 0])
    assert flog.log_f32(np.float32(1.0)) == 0.0
    # exact at powers of two up to the split of ln 2
    assert abs(float(flog.log_f32(np.float32(2.0)).item()) - math.log(2.0)) < 6e-8


def test_log_constants_are_rounded_rationals():
    from fractions import Fraction
    for c, (p, q) in ((flog.C3, (2, 3)), (flog.C5, (2, 5)), (flog.C7, (2, 7)),
                      (flog.C9, (2, 9)), (flog.C11, (2, 11))):
        exact = Fraction(p, q)
        v = Fraction(float(c))
        lo = Fraction(float(np.nextafter(c, np.float32(0))))
        hi = Fraction(float(np.nextafter(c, np.float32(1))))
        assert abs(v - exact) <= abs(lo - exact) and abs(v - exact) <= abs(hi - exact)
    # LN2_HI has at most 16 fractional bits, so e * LN2_HI is exact for |e| < 256
    assert float(flog.LN2_HI) * 65536 == int(float(flog.LN2_HI) * 65536)
    assert abs(float(flog.LN2_HI) + float(flog.LN2_LO) - math.log(2.0)) < 1e-13


def test_uniform_words_exact_and_symmetric():
    r = np.array([0, 0x1FF, 0x200, 0xFFFFFFFF, 0x80000000], dtype=np.uint32)
    u = flog.uniform_f32(r).astype(np.float64)
    assert u[0] == 2.0 ** -24 and u[1] == 2.0 ** -24
    assert u[2] == 3 * 2.0 ** -24
    assert u[3] == 1.0 - 2.0 ** -24
    assert u[4] == 0.5 + 2.0 ** -24


def test_gumbel_transform_accuracy():
    # every 23-bit level is reachable; sweep a dense subset plus the extremes
    levels = np.concatenate([np.arange(0, 1 << 23, 97, dtype=np.uint64),
                             np.arange((1 << 23) - 2048, 1 << 23, dtype=np.uint64),
                             np.arange(0, 2048, dtype=np.uint64)])
    r = (levels << np.uint64(9)).astype(np.uint32)
    u32 = flog.uniform_f32(r)
    g32 = flog.gumbel_f32(u32).astype(np.float64)
    u = u32.astype(np.float64)
    g64 = -np.log(-np.log(u))
    err = np.abs(g32 - g64)
    # absolute error bound relative to the Gumbel scale (|g| < 17)
    assert err.max() < 4e-6, err.max()
    # monotone in u, as -ln(-ln u) is
    order = np.argsort(u)
    assert np.all(np.diff(g32[order]) >= 0)


def test_gumbel_noise_is_nondecreasing_over_every_word_and_its_maximum():
    # The sampler's group bound relies on two facts about the specified noise
    # g32: it never decreases as the Philox word grows, and its largest value
    # (u = 1 - 2^-24) is the constant the CUDA screen uses.  Both are checked
    # here over all 2^23 distinct uniforms.
    import os
    import re
    r = (np.arange(1 << 23, dtype=np.uint64) << np.uint64(9)).astype(np.uint32)
    g = flog.gumbel_f32(flog.uniform_f32(r))
    assert np.all(np.diff(g) >= 0)
    src = open(os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                            "block_canvas_denoising_b200", "csrc", "dg_device.cuh")).read()
    m = re.search(r"kGumbelMaxNoise\s*=\s*([0-9.]+)f", src)
    assert m is not None
    assert np.float32(m.group(1)) == g.max()
