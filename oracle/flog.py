"""The float32 Gumbel transform the sampler's keys are defined with.

The denoising step draws its token by Gumbel-max (argmax of x + g with
g = -ln(-ln u)).  So that a replay of the sampler on the device's float32
logits reproduces the device's tokens bit for bit, the float32 key is
specified here with IEEE-754 operations only (correctly rounded add, sub,
mul, div; no fused multiply-add, no library ``log``):

``L(y)``, natural log of a positive normal float32 y:
  * split ``y = 2^e * m`` with m in [1, 2); if m > sqrt(2) halve m and
    increment e, so m lies in [sqrt(2)/2, sqrt(2)];
  * ``f = m - 1`` (exact), ``s = f / (m + 1)``, ``z = s*s``;
  * ``ln m = 2*atanh(s) = 2s + s*z*(2/3 + z*(2/5 + z*(2/7 + z*(2/9 + z*2/11))))``
    -- the odd series of atanh (Abramowitz & Stegun 4.5.64 via
    ln m = 2 atanh((m-1)/(m+1))), evaluated innermost first;
  * ``L = e*LN2_HI + (ln m + e*LN2_LO)`` where LN2_HI is ln 2 truncated to
    16 fractional bits (so e*LN2_HI is exact) and LN2_LO = RN(ln 2 - LN2_HI).

Every constant is the float32 round-to-nearest of the stated rational.

``u(r)``: the uniform of a 32-bit Philox word r is ``(2*(r >> 9) + 1) * 2^-24``,
an odd multiple of 2^-24 in (0, 1), exact in float32.

``g32(u) = -L(-L(u))`` and the key of vocabulary entry v is
``fl32(fl32(z_v * inv_tau) + g32(u_v))``.

TEST INFRASTRUCTURE: part of the CPU oracle (see ``oracle/__init__``).
"""
from __future__ import annotations

import math

import numpy as np

F32 = np.float32

C3 = F32(2.0 / 3.0)
C5 = F32(2.0 / 5.0)
C7 = F32(2.0 / 7.0)
C9 = F32(2.0 / 9.0)
C11 = F32(2.0 / 11.0)
LN2_HI = F32(math.floor(math.log(2.0) * 65536.0) / 65536.0)
LN2_LO = F32(math.log(2.0) - float(LN2_HI))
_SQRT2_MANT = np.uint32(0x3504F3)   # mantissa bits of float32(sqrt(2)) (rounded down)


def log_f32(y) -> np.ndarray:
    """L(y) as specified above, elementwise on positive normal float32."""
    y = np.ascontiguousarray(y, dtype=np.float32)
    b = y.view(np.uint32)
    e = ((b >> np.uint32(23)) & np.uint32(0xFF)).astype(np.int32) - 127
    mant = b & np.uint32(0x7FFFFF)
    m = (mant | np.uint32(0x3F800000)).view(np.float32)
    big = mant > _SQRT2_MANT
    m = np.where(big, m * F32(0.5), m).astype(np.float32)
    e = np.where(big, e + 1, e)
    f = m - F32(1.0)
    s = f / (m + F32(1.0))
    z = s * s
    r = z * C11
    r = C9 + r
    r = z * r
    r = C7 + r
    r = z * r
    r = C5 + r
    r = z * r
    r = C3 + r
    r = z * r
    lnm = (s + s) + s * r
    ef = e.astype(np.float32)
    return (ef * LN2_HI + (lnm + ef * LN2_LO)).astype(np.float32)


def uniform_f32(r) -> np.ndarray:
    """u = (2*(r >> 9) + 1) * 2^-24 from 32-bit words, as float32 (exact)."""
    r = np.asarray(r, dtype=np.uint32)
    odd = (r >> np.uint32(9)).astype(np.int64) * 2 + 1
    return odd.astype(np.float32) * F32(2.0 ** -24)


def gumbel_f32(u) -> np.ndarray:
    """g32(u) = -L(-L(u)) for u in (0, 1)."""
    u = np.asarray(u, dtype=np.float32)
    return -log_f32(-log_f32(u))
