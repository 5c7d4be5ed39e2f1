"""Seeded synthetic inputs for the denoising step.

This module is the one piece shared by the CPU oracle, the CUDA parity tests
and the bench.  It only *makes inputs*: random hidden states, a random tied
embedder, a random canvas, per-canvas step indices and the stand-in hidden
state of the adaptive loop.  It holds none of the arithmetic of the denoising
step itself (no logits, softmax, entropy, sampling, selection or stopping).

Everything is returned as raw bits (bf16 as ``uint16``, FP8-E4M3 as
``uint8``) so that both sides decode the same bytes with their own code.

Workload shapes follow the pages: a 256-slot canvas ("DiffusionGemma
Technical Report", abstract and Figure 4), a 262,144-token vocabulary and a
740M-parameter embedder, hence d = 2816 ("DiffusionGemma Technical Report",
Table 1).  The value distributions (h ~ N(0,1), E ~ N(0, 0.02^2)) are this
project's synthetic stand-ins; the pages publish no weights.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

__all__ = [
    "bf16_bits_from_f32", "bf16_bits_to_f32", "normal_bf16", "hidden_normal",
    "embedder_normal", "canvas_uniform", "step_indices_uniform",
    "quantize_e4m3_rows", "e4m3_bits_from_f32", "loop_targets", "loop_hidden", "block_targets",
]

# Rows generated per independent random stream.  Each chunk of rows draws from
# its own ``default_rng([seed, chunk])`` stream so chunks can be generated in
# parallel and the result does not depend on the thread count.
_CHUNK_ROWS = 4096


def bf16_bits_from_f32(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round to nearest, ties to even).

    Returns the 16-bit patterns as ``uint16``.  NaN inputs are not expected.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    b = x.view(np.uint32)
    rounding = np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))
    return ((b + rounding) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns to float32 (exact)."""
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def normal_bf16(rows: int, cols: int, seed: int, std: float) -> np.ndarray:
    """``rows x cols`` samples of N(0, std^2), rounded to bf16 bits.

    Row chunk ``c`` (rows ``c*4096 ...``) uses the stream
    ``np.random.default_rng([seed, c])``; samples are drawn in float32,
    scaled by ``float32(std)`` and rounded to nearest-even bf16.
    """
    out = np.empty((rows, cols), dtype=np.uint16)
    n_chunks = (rows + _CHUNK_ROWS - 1) // _CHUNK_ROWS
    s = np.float32(std)

    def work(c: int) -> None:
        r0 = c * _CHUNK_ROWS
        r1 = min(rows, r0 + _CHUNK_ROWS)
        g = np.random.default_rng([seed, c])
        x = g.standard_normal((r1 - r0, cols), dtype=np.float32)
        x *= s
        out[r0:r1] = bf16_bits_from_f32(x)

    if n_chunks == 1:
        work(0)
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(work, range(n_chunks)))
    return out


def hidden_normal(B: int, L: int, d: int, seed: int = 2) -> np.ndarray:
    """Canvas hidden states h[B*L, d] ~ N(0,1) as bf16 bits."""
    return normal_bf16(B * L, d, seed, 1.0)


def embedder_normal(V: int, d: int, seed: int = 1, std: float = 0.02) -> np.ndarray:
    """Tied embedder E[V, d] ~ N(0, 0.02^2) as bf16 bits."""
    return normal_bf16(V, d, seed, std)


def canvas_uniform(B: int, L: int, V: int, seed: int = 0) -> np.ndarray:
    """Initial canvas tokens, uniform in [0, V), int32 [B*L]."""
    g = np.random.default_rng(seed)
    return g.integers(0, V, size=B * L, dtype=np.int64).astype(np.int32)


def step_indices_uniform(B: int, max_steps: int, seed: int = 5) -> np.ndarray:
    """One step index per canvas, uniform in [0, max_steps - 1], int32 [B]."""
    g = np.random.default_rng(seed)
    return g.integers(0, max_steps, size=B, dtype=np.int64).astype(np.int32)


# ---------------------------------------------------------------------------
# FP8-E4M3 (OCP "E4M3FN": 1 sign, 4 exponent bits with bias 7, 3 mantissa
# bits, no infinities, max finite 448).  Encoding is input preparation only:
# both sides consume the same bytes and decode them with their own code.
# ---------------------------------------------------------------------------

def e4m3_bits_from_f32(x: np.ndarray) -> np.ndarray:
    """Encode float32 values (|x| <= 448) to E4M3 bits, round to nearest even.

    Values beyond +-448 saturate to +-448.  Written from the format
    definition: normal numbers 1.mmm * 2^(e-7) for e in 1..15 (e=15, m=7 is
    NaN and never produced), subnormals 0.mmm * 2^-6.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    sign = (x.view(np.uint32) >> np.uint32(31)).astype(np.uint8) << np.uint8(7)
    a = np.minimum(np.abs(x).astype(np.float64), 448.0)
    out = np.zeros(a.shape, dtype=np.uint8)
    nz = a > 0
    # exponent of the value, clamped to the subnormal range
    e = np.zeros(a.shape, dtype=np.int64)
    e[nz] = np.floor(np.log2(a[nz])).astype(np.int64)
    # correct floor(log2) rounding at exact powers of two
    e = np.where(nz & (np.ldexp(1.0, e) > a), e - 1, e)
    e = np.where(nz & (np.ldexp(1.0, e + 1) <= a), e + 1, e)
    e = np.maximum(e, -6)
    # quantum of the 3-bit mantissa at this exponent
    q = np.ldexp(1.0, e - 3)
    n = a / q                                   # exact in fp64
    n_rounded = np.round(n)                     # numpy rounds half to even
    n_int = n_rounded.astype(np.int64)          # 0..16
    # renormalise when rounding carried into the next binade
    carry = n_int >= 16
    e = np.where(carry, e + 1, e)
    n_int = np.where(carry, n_int // 2, n_int)
    # subnormal iff the leading bit is absent (e == -6 and n < 8)
    sub = n_int < 8
    exp_field = np.where(sub, 0, e + 7)
    man_field = np.where(sub, n_int, n_int - 8)
    code = (exp_field << 3) | man_field
    out = np.where(nz, code, 0).astype(np.uint8)
    return out | sign


def quantize_e4m3_rows(E_bits_bf16: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Per-row FP8-E4M3 quantisation of a bf16 embedder.

    For each vocabulary row v: ``s_v = float32(absmax_v) / 448`` (float32
    division; ``s_v = 1`` for an all-zero row), ``q_v = E4M3(E_v / s_v)``
    with the division in float32 and round-to-nearest-even, saturating at
    +-448.  Returns ``(q uint8 [V, d], s float32 [V])``.
    """
    V, d = E_bits_bf16.shape
    q = np.empty((V, d), dtype=np.uint8)
    s = np.empty(V, dtype=np.float32)
    step = 8192

    def work(r0: int) -> None:
        r1 = min(V, r0 + step)
        e = bf16_bits_to_f32(E_bits_bf16[r0:r1])
        amax = np.max(np.abs(e), axis=1)
        sc = np.where(amax > 0, amax / np.float32(448.0), np.float32(1.0)).astype(np.float32)
        s[r0:r1] = sc
        q[r0:r1] = e4m3_bits_from_f32(e / sc[:, None])

    with ThreadPoolExecutor(_threads()) as ex:
        list(ex.map(work, range(0, V, step)))
    return q, s


# ---------------------------------------------------------------------------
# Stand-in for the denoiser forward in the adaptive loop.
# ---------------------------------------------------------------------------

def loop_targets(L: int, V: int, seed: int = 3, B: int = 1) -> np.ndarray:
    """Target tokens y[B*L] the synthetic hidden states point towards."""
    g = np.random.default_rng(seed)
    return g.integers(0, V, size=B * L, dtype=np.int64).astype(np.int32)


def loop_hidden(k: int, y: np.ndarray, E_bits_bf16: np.ndarray, seed: int = 4) -> np.ndarray:
    """Synthetic hidden state of loop step k, as bf16 bits [len(y), d].

    ``h_i = (k/12) * 3 * E[y_i] / ||E[y_i]|| * sqrt(d) + n_i`` with
    ``n_i ~ N(0, 1)`` redrawn every step from ``default_rng([seed, k])``;
    computed in float64 and rounded to bf16.  It stands in for the model's
    forward pass, which the pages do not give: the signal grows with k so the
    per-slot entropy falls step by step.
    """
    d = E_bits_bf16.shape[1]
    Ey = bf16_bits_to_f32(E_bits_bf16[np.asarray(y, dtype=np.int64)]).astype(np.float64)
    norm = np.sqrt(np.sum(Ey * Ey, axis=1, keepdims=True))
    norm = np.where(norm > 0, norm, 1.0)
    g = np.random.default_rng([seed, int(k)])
    noise = g.standard_normal((len(y), d))
    h = (k / 12.0) * 3.0 * Ey / norm * math.sqrt(d) + noise
    return bf16_bits_from_f32(h.astype(np.float32))


def block_targets(j: int, committed: np.ndarray, L: int, V: int, B: int = 1, seed: int = 3) -> np.ndarray:
    """Targets y[B*L] of the stand-in hidden states of canvas block j in a
    block-by-block generation.

    Block 0 takes ``loop_targets``; block j >= 1 derives its targets from
    the block committed just before it, y_i = (c_i * 7919 + 104729 (i + 1)
    + j) mod V, so every block depends on what the previous one committed.
    (A stand-in for the model conditioning the next block on the appended
    context; the pages give no model to run.)
    """
    if j == 0:
        return loop_targets(L, V, seed=seed, B=B)
    c = np.asarray(committed[j - 1], dtype=np.int64)
    i = np.arange(B * L, dtype=np.int64)
    return ((c * 7919 + 104729 * (i + 1) + j) % V).astype(np.int32)
