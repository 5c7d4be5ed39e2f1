"""Pins of the self-conditioning oracle (the expected embedding
softmax(z / tau) E), against closed forms and a plain loop in exact
arithmetic."""
import math
from fractions import Fraction

import numpy as np

import synth
from oracle import selfcond, step


def test_uniform_logits_give_the_mean_embedding():
    # h = 0: every logit is 0, the tempered distribution is uniform
    V, d = 64, 16
    E = synth.embedder_normal(V, d, seed=1)
    h = np.zeros((3, d), np.uint16)
    got = selfcond.expected_embedding(h, E_bits=E, k=5)
    want = step.decode_bf16(E).mean(axis=0)
    assert np.allclose(got, want[None, :], rtol=0, atol=1e-15)


def test_dominant_logit_gives_that_row():
    # one logit far above the rest: the signal is that row of E
    V, d = 256, 32
    E = synth.embedder_normal(V, d, seed=2)
    e = step.decode_bf16(E)
    y = 77
    h = synth.bf16_bits_from_f32((60.0 * e[y] / np.linalg.norm(e[y]) * math.sqrt(d)).astype(np.float32))[None, :]
    got = selfcond.expected_embedding(h, E_bits=E, k=47)
    assert np.abs(got[0] - e[y]).max() < 1e-12


def test_matches_exact_rational_sum_on_a_tiny_case():
    # weights e^{x_v - max} evaluated in float64, then the weighted mean of
    # the rows formed exactly with fractions: the oracle must agree to
    # float64 rounding (a dropped term, a wrong normaliser, a transposed
    # operand or a missing temperature would not)
    V, d = 7, 5
    E = synth.embedder_normal(V, d, seed=3, std=0.5)
    h = synth.hidden_normal(1, 1, d, seed=4)
    k = 20
    tau = step.temperature(k)
    z = step.decode_bf16(h) @ step.decode_bf16(E).T
    x = z[0] / tau
    w = [Fraction(math.exp(xv - x.max())) for xv in x]
    Ef = [[Fraction(float(v)) for v in row] for row in step.decode_bf16(E)]
    den = sum(w)
    want = [float(sum(w[v] * Ef[v][j] for v in range(V)) / den) for j in range(d)]
    got = selfcond.expected_embedding(h, E_bits=E, k=k)[0]
    assert np.allclose(got, want, rtol=1e-13, atol=1e-15)


def test_temperature_sharpens_toward_the_argmax_row():
    V, d = 512, 24
    E = synth.embedder_normal(V, d, seed=5, std=0.3)
    h = synth.hidden_normal(1, 1, d, seed=6)
    e = step.decode_bf16(E)
    top = int(np.argmax(step.decode_bf16(h) @ e.T))
    dist = [np.linalg.norm(selfcond.expected_embedding(h, E_bits=E, k=k)[0] - e[top]) for k in (0, 23, 47)]
    assert dist[0] > dist[1] > dist[2]


def test_fp8_embedder_uses_the_dequantised_rows():
    V, d = 128, 16
    E = synth.embedder_normal(V, d, seed=7)
    q, s = synth.quantize_e4m3_rows(E)
    h = synth.hidden_normal(1, 2, d, seed=8)
    got = selfcond.expected_embedding(h, q=q, s=s, k=10)
    Ed = step.decode_e4m3(q) * s.astype(np.float64)[:, None]
    x = (step.decode_bf16(h) @ Ed.T) / step.temperature(10)
    p = np.exp(x - x.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    assert np.allclose(got, p @ Ed, rtol=0, atol=1e-15)


def test_abs_values_scale_bounds_the_signal():
    # sum_v p_v |E[v]| >= |sum_v p_v E[v]| elementwise, with equality where
    # E's column has one sign; for a non-negative embedder the two agree
    V, d = 512, 32
    E = synth.embedder_normal(V, d, seed=4)
    h = synth.hidden_normal(1, 4, d, seed=5)
    s_ = selfcond.expected_embedding(h, E_bits=E, k=3)
    a_ = selfcond.expected_embedding(h, E_bits=E, k=3, abs_values=True)
    assert np.all(a_ >= np.abs(s_) - 1e-15) and np.any(a_ > np.abs(s_) + 1e-6)
    Epos = (np.asarray(E, np.uint16) & np.uint16(0x7FFF)).astype(np.uint16)
    assert np.allclose(selfcond.expected_embedding(h, E_bits=Epos, k=3),
                       selfcond.expected_embedding(h, E_bits=Epos, k=3, abs_values=True), rtol=0, atol=1e-15)
