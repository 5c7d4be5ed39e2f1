"""Pins for the oracle's step functions against closed forms, exact
arithmetic, independent library routines, invariants and the pages' values."""
import json
import math
import os
from decimal import Decimal, getcontext
from fractions import Fraction

import numpy as np
import pytest
import torch

import synth
from oracle import step as S
from oracle.philox import split_seed
from oracle.replay import replay_step

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _chi2_pvalue(counts, expected):
    from scipy.stats import chi2
    m = expected > 0
    stat = float(np.sum((counts[m] - expected[m]) ** 2 / expected[m]))
    return chi2.sf(stat, int(m.sum()) - 1)


# ---- the pages' printed values ---------------------------------------------

def test_serving_defaults_match_pages():
    g = json.load(open(os.path.join(GOLDEN, "serving_defaults.json")))
    assert S.MAX_STEPS == g["max_denoising_steps"]["value"]
    assert S.TAU0 == g["temperature_start"]["value"]
    assert S.TAU1 == g["temperature_end"]["value"]
    assert S.STOP_ENTROPY == g["stop_entropy_threshold"]["value"]
    assert S.ENTROPY_BOUND == g["selection_entropy_bound"]["value"]
    # d = 2816 is the multiple of 64 that the 740M embedder over 262,144
    # tokens implies (740e6 / 262144 = 2822.9)
    d = 740e6 / 262144
    assert abs(d - 2816) < 16 and 2816 % 64 == 0
    assert abs(262144 - g["vocabulary_tokens_approx"]["value"]) / 262144 < 0.01


# ---- a1 temperature -----------------------------------------------------------

def test_temperature_endpoints_and_linearity():
    assert S.temperature(0) == 0.8
    assert S.temperature(47) == 0.4
    for k in range(48):
        assert abs(S.temperature(k) - (0.8 - 0.4 * k / 47)) < 1e-15
    assert S.temperature(0, max_steps=1) == 0.8
    with pytest.raises(ValueError):
        S.temperature(48)
    assert S.inv_tau_f32(0) == np.float32(1.25)
    assert S.inv_tau_f32(47) == np.float32(2.5)


# ---- decoding (vs torch's independent converters) -----------------------------

def test_bf16_decode_matches_torch():
    bits = np.arange(0, 65536, dtype=np.uint32).astype(np.uint16)
    t = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).float().numpy()
    mine = S.decode_bf16(bits)
    fin = np.isfinite(t)
    assert np.array_equal(mine[fin], t[fin].astype(np.float64))


def test_bf16_encode_matches_torch():
    x = np.random.default_rng(3).standard_normal(100000).astype(np.float32) * 7
    mine = synth.bf16_bits_from_f32(x)
    t = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(mine, t)


def test_e4m3_decode_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    t = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    mine = S.decode_e4m3(codes)
    fin = np.isfinite(t)
    assert np.array_equal(np.isfinite(mine), fin)
    assert np.array_equal(mine[fin], t[fin])


def test_e4m3_encode_matches_torch():
    g = np.random.default_rng(4)
    x = np.concatenate([g.uniform(-448, 448, 50000), g.standard_normal(50000) * 0.01,
                        S.decode_e4m3(np.arange(256, dtype=np.uint8)[np.arange(256) % 128 != 127])]
                       ).astype(np.float32)
    mine = synth.e4m3_bits_from_f32(x)
    t = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    # torch may encode -0.0 and 0.0 identically; compare decoded values
    assert np.array_equal(S.decode_e4m3(mine), S.decode_e4m3(t))


def test_row_quantisation_roundtrip():
    E = synth.embedder_normal(64, 128, seed=9)
    q, s = synth.quantize_e4m3_rows(E)
    deq = S.dequantized_embedder(q=q, s=s)
    ref = S.decode_bf16(E)
    amax = np.abs(ref).max(axis=1)
    # E4M3 has a 3-bit mantissa: relative error <= 2^-4 of the row's scale
    assert np.all(np.abs(deq - ref) <= amax[:, None] * 2.0 ** -4 / 448 * 256 + 1e-12)
    assert np.allclose(np.abs(deq).max(axis=1), amax, rtol=2 ** -4)


# ---- a2 logits -------------------------------------------------------------------

def test_logits_match_exact_rational_dot_products():
    h = synth.normal_bf16(3, 24, seed=21, std=1.0)
    E = synth.normal_bf16(11, 24, seed=22, std=0.3)
    z = S.logits(h, E_bits=E, v_chunk=4)
    hf = [[Fraction(float(v)) for v in row] for row in S.decode_bf16(h)]
    Ef = [[Fraction(float(v)) for v in row] for row in S.decode_bf16(E)]
    for r in range(3):
        for v in range(11):
            exact = sum(a * b for a, b in zip(hf[r], Ef[v]))
            assert abs(z[r, v] - float(exact)) <= 1e-12 * max(1.0, abs(float(exact)))


def test_fp8_logits_factor_the_row_scale():
    h = synth.normal_bf16(2, 32, seed=23, std=1.0)
    E = synth.normal_bf16(9, 32, seed=24, std=0.02)
    q, s = synth.quantize_e4m3_rows(E)
    z = S.logits(h, q=q, s=s)
    ref = S.decode_bf16(h) @ (S.decode_e4m3(q).T) * s.astype(np.float64)[None, :]
    assert np.allclose(z, ref, rtol=1e-14, atol=1e-14)


# ---- a3 entropy ------------------------------------------------------------------

def test_entropy_constant_logits_is_log_v():
    for V in (2, 16, 8192):
        x = np.full((2, V), 3.25)
        assert np.allclose(S.entropy(x), math.log(V), rtol=0, atol=1e-12)


def test_entropy_one_hot_is_zero():
    x = np.zeros((1, 64))
    x[0, 17] = 900.0
    assert S.entropy(x)[0] == 0.0


def test_entropy_matches_high_precision_enumeration():
    getcontext().prec = 60
    g = np.random.default_rng(5)
    for V in (2, 3, 7, 16):
        x = g.standard_normal((4, V)) * 3
        H = S.entropy(x)
        for r in range(4):
            xs = [Decimal(float(v)) for v in x[r]]
            Z = sum(v.exp() for v in xs)
            p = [v.exp() / Z for v in xs]
            Hx = -sum(pi * pi.ln() for pi in p)
            assert abs(H[r] - float(Hx)) < 1e-13


def test_entropy_shift_invariant_and_temperature_monotone():
    x = np.random.default_rng(6).standard_normal((3, 500))
    assert np.allclose(S.entropy(x), S.entropy(x + 123.0), atol=1e-12)
    # a lower temperature sharpens the distribution
    assert np.all(S.entropy(x / 0.4) < S.entropy(x / 0.8))


# ---- a4 argmax -------------------------------------------------------------------

def test_argmax_ties_to_lowest():
    a = np.array([[1.0, 5.0, 5.0, 2.0], [7.0, 7.0, 7.0, 7.0]])
    assert list(S.argmax_lowest(a)) == [1, 0]


# ---- a5 Gumbel-max draw ------------------------------------------------------------

def _draws(x, n_canvas, key_fn):
    V = x.shape[0]
    toks = []
    for b in range(n_canvas):
        w = S.gumbel_words(np.arange(0, 65536, dtype=np.uint64), b, 3, V, seed=777)
        toks.append(key_fn(np.broadcast_to(x, (65536, V)), w))
    return np.concatenate(toks)


def test_gumbel_max_samples_softmax_f64():
    x = np.array([0.0, 1.0, -0.5, 2.0, 0.3, -2.0, 1.5, 0.0, -1.0, 0.7, 0.2, -0.3, 1.1, -1.7, 0.4, 0.9])
    toks = _draws(x, 16, lambda xx, w: S.gumbel_sample(xx, w)[0])
    p = np.exp(x - x.max())
    p /= p.sum()
    counts = np.bincount(toks, minlength=16).astype(np.float64)
    assert _chi2_pvalue(counts, p * len(toks)) > 1e-4


def test_gumbel_max_samples_softmax_f32_key():
    from oracle.replay import key_f32
    x = np.array([0.5, -1.0, 1.25, 0.0, 2.0, -0.25, 0.75, 1.0], dtype=np.float32)
    it = np.float32(1.0)
    toks = _draws(x, 8, lambda xx, w: np.argmax(key_f32(xx, it, w), axis=1))
    p = np.exp(x.astype(np.float64) - x.max())
    p /= p.sum()
    counts = np.bincount(toks, minlength=8).astype(np.float64)
    assert _chi2_pvalue(counts, p * len(toks)) > 1e-4


def test_gumbel_wrong_sign_would_fail():
    # a transform with a flipped sign samples softmax(-x); the chi-square
    # test above must reject it, so it can catch that mistake
    x = np.array([0.0, 1.0, 2.0, 3.0])
    w = S.gumbel_words(np.arange(0, 65536, dtype=np.uint64), 0, 1, 4, seed=5)
    u = S.uniform_f64(w)
    bad = np.argmax(np.broadcast_to(x, (65536, 4)) + np.log(-np.log(u)), axis=1)
    p = np.exp(x - x.max())
    p /= p.sum()
    counts = np.bincount(bad, minlength=4).astype(np.float64)
    assert _chi2_pvalue(counts, p * len(bad)) < 1e-6


# ---- a7 selection -------------------------------------------------------------------

def test_select_hand_case():
    H = np.array([0.05, 0.01, 0.2, 0.03])
    acc, n, _ = S.select(H, 0.1)
    assert n == 3 and list(acc) == [1, 1, 0, 1]


def test_select_at_least_one_and_ties_to_lower_slot():
    acc, n, _ = S.select(np.array([0.5, 0.5, 0.5]), 0.1)
    assert n == 1 and list(acc) == [1, 0, 0]


def test_select_all_zero_entropy_accepts_all():
    acc, n, _ = S.select(np.zeros(256), 0.1)
    assert n == 256 and acc.all()


def test_select_monotone_in_bound():
    g = np.random.default_rng(8)
    for _ in range(50):
        H = g.exponential(0.02, 256)
        prev = np.zeros(256, np.uint8)
        for bound in (0.0, 0.01, 0.05, 0.1, 0.3, 1.0, 10.0):
            acc, _, _ = S.select(H, bound)
            assert np.all(acc >= prev)
            prev = acc


def test_select_inclusive_threshold():
    acc, n, _ = S.select(np.array([0.0625, 0.0625, 0.25]), 0.125)
    assert n == 2   # 0.0625 + 0.0625 == 0.125 exactly, inclusive


# ---- a8 renoise ------------------------------------------------------------------------

def test_renoise_uniform_over_vocabulary():
    V = 8192
    toks = np.concatenate([S.renoise_tokens(b, k, 256, V, seed=31) for b in range(64) for k in range(48)])
    assert toks.min() >= 0 and toks.max() < V
    counts = np.bincount(toks, minlength=V).astype(np.float64)
    assert _chi2_pvalue(counts, np.full(V, len(toks) / V)) > 1e-4


def test_renoise_power_of_two_is_top_bits():
    from oracle.philox import philox4x32_10
    k0, k1 = split_seed(31)
    o = philox4x32_10(np.uint64(0), np.arange(256, dtype=np.uint64) | np.uint64(1 << 16),
                      np.uint64(2), np.uint64(1), k0, k1)
    assert np.array_equal(S.renoise_tokens(1, 2, 256, 1 << 18, 31), (o[0] >> np.uint32(14)).astype(np.int32))


# ---- a9 stop ----------------------------------------------------------------------------

def test_stop_rules():
    H0 = np.full(256, 1e-4)
    am = np.arange(256, dtype=np.int32)
    assert S.stop_flag(H0, am, am, True)[0]
    assert not S.stop_flag(H0, am, am, False)[0]          # first step never stops
    other = am.copy()
    other[7] += 1
    assert not S.stop_flag(H0, am, other, True)[0]        # predictions changed
    assert not S.stop_flag(np.full(256, 0.005), am, am, True)[0]   # strict threshold


# ---- composed step ---------------------------------------------------------------------------

def _tiny_inputs(B=2, L=256, d=128, V=512):
    h = synth.hidden_normal(B, L, d, seed=2)
    E = synth.embedder_normal(V, d, seed=1)
    return h, E


def test_step_composition_invariants():
    B, L, V = 2, 256, 512
    h, E = _tiny_inputs(B, L, 128, V)
    r = S.denoise_step(h, E_bits=E, B=B, L=L, step_idx=np.array([0, 30]),
                       has_prev=np.zeros(B, np.uint8), prev_argmax=np.zeros(B * L, np.int32))
    for b in range(B):
        sl = slice(b * L, (b + 1) * L)
        noise = S.renoise_tokens(b, [0, 30][b], L, V, 1234)
        assert np.array_equal(r["canvas"][sl], np.where(r["accept"][sl] == 1, r["sampled"][sl], noise))
        assert r["accept"][sl].sum() == r["n_accept"][b] >= 1
    assert not r["stop"].any()
    assert np.all((r["sampled"] >= 0) & (r["sampled"] < V))
    assert np.all(r["entropy"] >= 0) and np.all(r["entropy"] <= math.log(V) + 1e-12)


def test_replay_of_rounded_logits_agrees_with_f64_draw():
    B, L, V = 1, 256, 512
    h, E = _tiny_inputs(B, L, 128, V)
    k = np.array([11])
    r64 = S.denoise_step(h, E_bits=E, B=B, L=L, step_idx=k, has_prev=np.zeros(1, np.uint8),
                         prev_argmax=np.zeros(L, np.int32))
    z32 = S.logits(h, E_bits=E).astype(np.float32)
    rr = replay_step(z32, B=B, L=L, step_idx=k, has_prev=np.zeros(1, np.uint8),
                     prev_argmax=np.zeros(L, np.int32))
    diff = rr["sampled"] != r64["sampled"]
    assert np.all(r64["gumbel_margin"][diff] < 1e-3)
    assert diff.mean() <= 0.01
    assert np.abs(rr["entropy"] - r64["entropy"]).max() < 1e-5


# ---- selection-rule variants ------------------------------------------------

def test_select_mi_rule_hand_case():
    from oracle.step import SELECT_MI, SELECT_CUMSUM
    H = np.array([0.05, 0.02, 0.03, 0.5, 0.01])
    # sorted 0.01 (s4), 0.02 (s1), 0.03 (s2), 0.05 (s0), 0.5 (s3); the sum of a
    # prefix minus its largest entropy is 0, 0.01, 0.03, 0.06, 0.11
    acc, n, _ = S.select(H, 0.1, SELECT_MI)
    assert n == 4 and acc.tolist() == [1, 1, 1, 0, 1]
    acc_c, n_c, _ = S.select(H, 0.1, SELECT_CUMSUM)
    assert n_c == 3 and acc_c.tolist() == [0, 1, 1, 0, 1]


def test_select_mi_rule_brute_force_definition():
    # longest prefix of the (entropy, slot) order whose sum minus its largest
    # entropy is <= bound, by plain loops over every prefix
    from oracle.step import SELECT_MI
    rng = np.random.default_rng(17)
    for trial in range(300):
        L = int(rng.integers(1, 9))
        H = rng.exponential(0.04, L) * (rng.random(L) < 0.8)
        bound = float(rng.choice([0.0, 0.01, 0.05, 0.1, 0.3]))
        order = sorted(range(L), key=lambda i: (H[i], i))
        best = 0
        for n in range(1, L + 1):
            pre = [H[i] for i in order[:n]]
            if sum(pre) - max(pre) <= bound:
                best = n
        want = np.zeros(L, np.uint8)
        want[order[:best]] = 1
        acc, n, _ = S.select(H, bound, SELECT_MI)
        assert n == best and np.array_equal(acc, want), (trial, H, bound)


def test_select_mi_contains_cumsum_and_is_monotone():
    from oracle.step import SELECT_MI, SELECT_CUMSUM
    rng = np.random.default_rng(5)
    for _ in range(100):
        H = rng.exponential(0.02, 256)
        a_c, _, _ = S.select(H, 0.1, SELECT_CUMSUM)
        a_m, _, _ = S.select(H, 0.1, SELECT_MI)
        assert np.all(a_m >= a_c)
        prev = 0
        for g in (0.0, 0.02, 0.05, 0.1, 0.2, 1.0):
            _, n, _ = S.select(H, g, SELECT_MI)
            assert n >= max(prev, 1)
            prev = n


def test_select_topk_rule():
    from oracle.step import SELECT_TOPK
    H = np.array([0.3, 0.1, 0.1, 0.0, 0.2])
    acc, n, m = S.select(H, 0.1, SELECT_TOPK, 3)
    assert n == 3 and acc.tolist() == [0, 1, 1, 1, 0]     # ties to the lower slot
    acc, n, m = S.select(np.zeros(6), 0.1, SELECT_TOPK, 2)
    assert acc.tolist() == [1, 1, 0, 0, 0, 0] and m == 0.0
    acc, n, _ = S.select(H, 0.1, SELECT_TOPK, 5)
    assert acc.sum() == 5
    with pytest.raises(ValueError):
        S.select(H, 0.1, SELECT_TOPK, 0)
