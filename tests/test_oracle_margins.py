"""Pins for the oracle's decision margins.

Every allowed GPU/oracle mismatch is excused by one of three oracle-side
margins (the Gumbel margin of a draw, the entropy-order margin of a
selection cut, the stop margin of a canvas), so each is checked here on
hand cases whose value follows from the definitions and can be worked out
on paper, and each check is shown to reject a plausible mistake planted in
a copy of the oracle function (a wrong neighbour, a dropped term, a wrong
sign).

Definitions (the decision margins of the tolerance accounting):
  * Gumbel margin: best key minus second-best key of the row;
  * order margin of a selection cut after n slots (sorted by entropy):
      cumulative-sum rule: min(|c_n - b|, |c_{n+1} - b|, H_(n+1) - H_(n));
      mutual-information rule: the same with the exclusive sums e_j;
      top-k: H_(k+1) - H_(k);
  * stop margin: |mean H - threshold|.
"""
import math

import numpy as np
import pytest

from oracle import step as S


def _word_for_u(u):
    """The Philox word whose u = (2 (r >> 9) + 1) 2^-24 is u (u must be of
    that form)."""
    q = int(round((u * 2.0 ** 24 - 1) / 2))
    assert (2 * q + 1) * 2.0 ** -24 == u
    return np.uint32(q << 9)


# ---------------------------------------------------------------------------
# Gumbel margin
# ---------------------------------------------------------------------------

U_MAX = 1.0 - 2.0 ** -24   # largest u: -ln u = 2^-24 + 2^-49 + ...
U_MIN = 2.0 ** -24         # smallest u: -ln u = 24 ln 2


def check_gumbel_margin(fn):
    # (1) the top two share one word: the noise cancels, margin = 0.25
    x = np.array([[1.25, 1.0, -100.0, -100.0]])
    w = np.array([[_word_for_u(0.5 + 2.0 ** -24)] * 2 + [_word_for_u(U_MIN)] * 2], dtype=np.uint32)
    tok, m = fn(x, w)
    assert tok[0] == 0 and abs(m[0] - 0.25) < 1e-12, (tok, m)
    # (2) equal logits, extreme words: g(U_MAX) = 24 ln 2 - 2^-25 + O(2^-50)
    #     and g(U_MIN) = -ln(24 ln 2), so the margin is
    #     24 ln 2 + ln(24 ln 2) - 2^-25, and the winner is the U_MAX slot
    x = np.zeros((1, 3))
    w = np.array([[_word_for_u(U_MIN), _word_for_u(U_MAX), _word_for_u(U_MIN)]], dtype=np.uint32)
    tok, m = fn(x, w)
    expect = 24 * math.log(2) + math.log(24 * math.log(2)) - 2.0 ** -25
    assert tok[0] == 1 and abs(m[0] - expect) < 1e-9, (tok, m, expect)
    # (3) a tie of keys (same logit, same word): margin 0, lowest index wins
    x = np.array([[0.5, 2.0, 2.0, 0.1]])
    w = np.array([[_word_for_u(0.25 + 2.0 ** -24)] * 4], dtype=np.uint32)
    tok, m = fn(x, w)
    assert tok[0] == 1 and m[0] == 0.0, (tok, m)


def test_gumbel_margin_hand_cases():
    check_gumbel_margin(S.gumbel_sample)


def test_gumbel_margin_check_rejects_planted_mistakes():
    def best_minus_worst(x, words):          # wrong neighbour
        key = x - np.log(-np.log(S.uniform_f64(words)))
        return np.argmax(key, axis=1).astype(np.int32), key.max(axis=1) - key.min(axis=1)

    def noise_sign_flipped(x, words):        # wrong sign of the Gumbel noise
        key = x + np.log(-np.log(S.uniform_f64(words)))
        top2 = -np.partition(-key, 1, axis=1)[:, :2]
        return np.argmax(key, axis=1).astype(np.int32), top2[:, 0] - top2[:, 1]

    for bad in (best_minus_worst, noise_sign_flipped):
        with pytest.raises(AssertionError):
            check_gumbel_margin(bad)


# ---------------------------------------------------------------------------
# Entropy-order margin of the selection cut
# ---------------------------------------------------------------------------

def check_select_margins(fn):
    # cumulative sums 0.01, 0.03, 0.06, 0.11, 0.61 against 0.1: n = 3;
    # |c_3 - b| = 0.04, |c_4 - b| = 0.01, gap H_(4) - H_(3) = 0.02
    H = np.array([0.05, 0.01, 0.5, 0.03, 0.02])
    acc, n, m = fn(H, 0.1, S.SELECT_CUMSUM, 1)
    assert n == 3 and list(acc) == [0, 1, 0, 1, 1] and abs(m - 0.01) < 1e-15, (n, acc, m)
    # the same entropies, exclusive sums 0, 0.01, 0.03, 0.06, 0.11: n = 4;
    # |e_4 - b| = 0.04, |e_5 - b| = 0.01, gap 0.45
    acc, n, m = fn(H, 0.1, S.SELECT_MI, 1)
    assert n == 4 and list(acc) == [1, 1, 0, 1, 1] and abs(m - 0.01) < 1e-15, (n, acc, m)
    # top-2: gap H_(3) - H_(2) = 0.01
    acc, n, m = fn(H, 0.1, S.SELECT_TOPK, 2)
    assert n == 2 and list(acc) == [0, 1, 0, 0, 1] and abs(m - 0.01) < 1e-15, (n, acc, m)
    # the entropy gap at the cut is the closest call: sums 0.02, 0.07,
    # 0.1200002: n = 2, |c_2 - b| = 0.03, |c_3 - b| = 0.0200002, gap 2e-7
    H = np.array([0.9, 0.0500002, 0.02, 0.05])
    acc, n, m = fn(H, 0.1, S.SELECT_CUMSUM, 1)
    assert n == 2 and list(acc) == [0, 0, 1, 1] and abs(m - 2e-7) < 1e-15, (n, acc, m)
    # the sum at the cut is the closest call: sums 0.0399, 0.0999, 0.1699:
    # n = 2, |c_2 - b| = 1e-4, |c_3 - b| = 0.0699, gap 0.01
    H = np.array([0.07, 0.0399, 0.06])
    acc, n, m = fn(H, 0.1, S.SELECT_CUMSUM, 1)
    assert n == 2 and abs(m - 1e-4) < 1e-15, (n, m)


def test_select_margin_hand_cases():
    check_select_margins(S.select)


def test_select_margin_check_rejects_planted_mistakes():
    def only_the_sum_before_the_cut(H, bound, rule, top_k):     # drops |c_{n+1} - b|
        acc, n, _ = S.select(H, bound, rule, top_k)
        Hs = np.sort(H)
        c = np.cumsum(Hs) if rule == S.SELECT_CUMSUM else np.concatenate([[0.0], np.cumsum(Hs)[:-1]])
        ms = [abs(c[n - 1] - bound)] if rule != S.SELECT_TOPK else []
        if n < len(H):
            ms.append(Hs[n] - Hs[n - 1])
        return acc, n, min(ms)

    def no_entropy_gap(H, bound, rule, top_k):                  # drops the gap term
        acc, n, _ = S.select(H, bound, rule, top_k)
        Hs = np.sort(H)
        c = np.cumsum(Hs) if rule == S.SELECT_CUMSUM else np.concatenate([[0.0], np.cumsum(Hs)[:-1]])
        ms = [abs(c[n - 1] - bound)] + ([abs(c[n] - bound)] if n < len(H) else [])
        return acc, n, min(ms) if rule != S.SELECT_TOPK else float("inf")

    def gap_on_the_wrong_side(H, bound, rule, top_k):           # H_(n) - H_(n-1)
        acc, n, m = S.select(H, bound, rule, top_k)
        Hs = np.sort(H)
        g = Hs[n - 1] - Hs[n - 2] if n >= 2 else float("inf")
        c = np.cumsum(Hs) if rule == S.SELECT_CUMSUM else np.concatenate([[0.0], np.cumsum(Hs)[:-1]])
        ms = [g]
        if rule != S.SELECT_TOPK:
            ms += [abs(c[n - 1] - bound)] + ([abs(c[n] - bound)] if n < len(H) else [])
        return acc, n, min(ms)

    for bad in (only_the_sum_before_the_cut, no_entropy_gap, gap_on_the_wrong_side):
        with pytest.raises(AssertionError):
            check_select_margins(bad)


# ---------------------------------------------------------------------------
# Stop margin
# ---------------------------------------------------------------------------

def check_stop_margin(fn):
    a = np.arange(8)
    # mean 0.004: below the threshold by 0.001
    st, m = fn(np.full(8, 0.004), a, a, True, 0.005)
    assert st and abs(m - 0.001) < 1e-15, (st, m)
    # mean 0.0075 (values 0.005 and 0.01): above by 0.0025, no stop
    st, m = fn(np.array([0.005, 0.01] * 4), a, a, True, 0.005)
    assert not st and abs(m - 0.0025) < 1e-15, (st, m)
    # the margin is that of the mean even when the prediction changed
    st, m = fn(np.full(8, 0.002), a, a[::-1], True, 0.005)
    assert not st and abs(m - 0.003) < 1e-15, (st, m)


def test_stop_margin_hand_cases():
    check_stop_margin(S.stop_flag)


def test_stop_margin_check_rejects_planted_mistakes():
    def max_instead_of_mean(H, am, prev, has_prev, thr):
        st, _ = S.stop_flag(H, am, prev, has_prev, thr)
        return st, abs(float(np.max(H)) - thr)

    def signed_margin(H, am, prev, has_prev, thr):
        st, _ = S.stop_flag(H, am, prev, has_prev, thr)
        return st, float(np.mean(H)) - thr

    for bad in (max_instead_of_mean, signed_margin):
        with pytest.raises(AssertionError):
            check_stop_margin(bad)
