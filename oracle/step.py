"""Plain float64 definition of one denoising step of the 256-slot canvas.

Each function states the passage of the pages it follows.  Pages are cited by
title and section:

* [Docs] "DiffusionGemma" (Google AI for Developers model docs), table
  "Recommended serving configuration" (rows: maximum denoising steps,
  temperature schedule, adaptive early stopping, token selection).
* [Report] "DiffusionGemma Technical Report" (arXiv:2608.00146, METAL MEDIA
  summary) -- Table 1 (262k vocabulary, 740M embedder), Figure 3 (uniform
  noise distribution), Figure 4 (denoising loop), Figure 9 (N sweep).
* [Press] "Google DiffusionGemma generates 256 tokens in parallel and
  self-corrects" (euno.news / VentureBeat), section "What DiffusionGemma does".
* [Review] "DiffusionGemma technical report review" (LLM Wiki / PyTorchKR),
  section "Key points" (self-correction).

Readings where the pages are silent (also listed in the design notes):
the selection rule is the cumulative-entropy prefix; entropy is that of the
temperature-scaled distribution in nats; tau runs from tau0 at k = 0 to tau1
at k = N-1; ties go to the lower index; renoise is uniform over [0, V).

TEST INFRASTRUCTURE: part of the CPU oracle (see ``oracle/__init__``).
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from .philox import philox4x32_10, split_seed

# Serving defaults, [Docs] "Recommended serving configuration".
TAU0 = 0.8            # temperature at the first step
TAU1 = 0.4            # temperature at the last step
MAX_STEPS = 48        # maximum denoising steps per canvas
ENTROPY_BOUND = 0.1   # token-selection entropy bound
STOP_ENTROPY = 0.005  # adaptive-stop mean-entropy threshold

PURPOSE_GUMBEL = 0
PURPOSE_RENOISE = 1
PURPOSE_INIT = 3      # the noise canvas a block starts from


# selection rules (the default is this project's reading of the pages)
SELECT_CUMSUM = 0   # longest sorted prefix with sum of entropies <= bound, at least one
SELECT_MI = 1       # longest sorted prefix with sum minus its largest entropy <= bound
SELECT_TOPK = 2     # the top_k lowest-entropy slots


@dataclass
class Params:
    tau0: float = TAU0
    tau1: float = TAU1
    max_steps: int = MAX_STEPS
    entropy_bound: float = ENTROPY_BOUND
    stop_entropy: float = STOP_ENTROPY
    seed: int = 1234
    selection_rule: int = SELECT_CUMSUM
    top_k: int = 1
    block: int = 0    # index of the canvas block in a block-by-block generation


def counter_step(k: int, block: int = 0) -> int:
    """Third Philox counter word of step k of canvas block ``block``:
    k | block << 16, so every block draws its own streams (k < 2^16).
    [Report] Figure 4: generation proceeds block after block, each block
    denoised from fresh noise; a single block is block 0 (word = k)."""
    if not (0 <= k < 1 << 16 and 0 <= block < 1 << 16):
        raise ValueError("step or block index out of range")
    return int(k) | (int(block) << 16)


# --------------------------------------------------------------------------
# decoding of the stored inputs
# --------------------------------------------------------------------------

def decode_bf16(bits) -> np.ndarray:
    """bfloat16 bit patterns -> float64 (exact): the pattern is the upper
    half of a float32."""
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    with np.errstate(invalid="ignore"):
        return b.view(np.float32).astype(np.float64)


def _e4m3_table() -> np.ndarray:
    # OCP FP8 E4M3FN: exponent bias 7, 3 mantissa bits, no infinities;
    # exponent field 0 encodes subnormals 0.mmm * 2^-6; code 0x7F is NaN.
    t = np.empty(256, dtype=np.float64)
    for code in range(256):
        sign = -1.0 if code & 0x80 else 1.0
        ef = (code >> 3) & 0xF
        mf = code & 0x7
        if ef == 0xF and mf == 0x7:
            t[code] = np.nan
        elif ef == 0:
            t[code] = sign * (mf / 8.0) * 2.0 ** -6
        else:
            t[code] = sign * (1.0 + mf / 8.0) * 2.0 ** (ef - 7)
    return t


_E4M3 = _e4m3_table()


def decode_e4m3(bits) -> np.ndarray:
    """FP8-E4M3 bit patterns -> float64 (exact)."""
    return _E4M3[np.asarray(bits, dtype=np.uint8)]


# --------------------------------------------------------------------------
# a1: temperature schedule
# --------------------------------------------------------------------------

def temperature(k: int, tau0: float = TAU0, tau1: float = TAU1, max_steps: int = MAX_STEPS) -> float:
    """Linear schedule from tau0 at step 0 to tau1 at step N-1.

    [Docs] temperature-schedule row: a linear decrease from 0.8 to 0.4, hot
    at the start and cool at the end; [Report] Figure 9: a larger N gives milder annealing, so the
    schedule spans the N steps.  For N = 1 the single step uses tau0.
    """
    if not 0 <= k < max_steps:
        raise ValueError("step index out of range")
    if max_steps == 1:
        return float(tau0)
    return float(tau0) - (float(tau0) - float(tau1)) * k / (max_steps - 1)


def inv_tau_f32(k: int, tau0: float = TAU0, tau1: float = TAU1, max_steps: int = MAX_STEPS) -> np.float32:
    """1/tau_k computed in float64 and rounded once to float32."""
    return np.float32(1.0 / temperature(k, tau0, tau1, max_steps))


# --------------------------------------------------------------------------
# a2: tied LM head
# --------------------------------------------------------------------------

def dequantized_embedder(E_bits=None, q=None, s=None) -> np.ndarray:
    """The embedder in float64: bf16 bits, or FP8-E4M3 codes times a per-row
    float32 scale."""
    if E_bits is not None:
        return decode_bf16(E_bits)
    return decode_e4m3(q) * np.asarray(s, dtype=np.float64)[:, None]


def logits(h_bits, E_bits=None, q=None, s=None, v_chunk: int = 8192) -> np.ndarray:
    """z = h . E^T in float64 (inputs decoded exactly), [rows, V].

    The head is tied to the 740M-parameter embedder over the 262k vocabulary
    ([Report] Table 1); no bias or soft-cap is stated.
    """
    h = decode_bf16(h_bits)
    V = (E_bits if E_bits is not None else q).shape[0]
    z = np.empty((h.shape[0], V), dtype=np.float64)
    for v0 in range(0, V, v_chunk):
        v1 = min(V, v0 + v_chunk)
        if E_bits is not None:
            Ec = decode_bf16(E_bits[v0:v1])
        else:
            Ec = decode_e4m3(q[v0:v1]) * np.asarray(s[v0:v1], dtype=np.float64)[:, None]
        z[:, v0:v1] = h @ Ec.T
    return z


# --------------------------------------------------------------------------
# a3 / a4: entropy of the tempered distribution, argmax prediction
# --------------------------------------------------------------------------

def entropy(x: np.ndarray) -> np.ndarray:
    """Entropy (nats) of softmax(x) per row, two-pass, clamped at 0.

    H = ln S - T/S with m = max x, S = sum e^(x-m), T = sum (x-m) e^(x-m);
    this equals -sum p ln p.  [Docs] the adaptive-stop and token-selection
    rows both use the model's entropy.
    """
    m = np.max(x, axis=1, keepdims=True)
    d = x - m
    e = np.exp(d)
    S = np.sum(e, axis=1)
    T = np.sum(d * e, axis=1)
    H = np.log(S) - T / S
    return np.maximum(H, 0.0)


def argmax_lowest(a: np.ndarray) -> np.ndarray:
    """Per-row argmax, ties to the lowest index (int32)."""
    return np.argmax(a, axis=1).astype(np.int32)


# --------------------------------------------------------------------------
# a5: Gumbel-max draw with a counter-based Philox stream
# --------------------------------------------------------------------------

def gumbel_words(slots, b: int, k: int, V: int, seed: int) -> np.ndarray:
    """Philox4x32-10 words for the Gumbel noise of the given slots of
    canvas b at step k: [len(slots), V] uint32.

    Counter (v >> 2, slot | purpose << 16, k, b), key (seed lo, seed hi),
    output lane v & 3, purpose 0.
    """
    slots = np.asarray(slots, dtype=np.uint64)
    k0, k1 = split_seed(seed)
    q = np.arange((V + 3) // 4, dtype=np.uint64)[None, :]
    c1 = (slots | np.uint64(PURPOSE_GUMBEL << 16))[:, None]
    o = philox4x32_10(q, c1, np.uint64(k), np.uint64(b), k0, k1)
    w = np.empty((len(slots), V), dtype=np.uint32)
    for lane in range(4):
        w[:, lane::4] = o[lane][:, :len(range(lane, V, 4))]
    return w


def uniform_f64(words) -> np.ndarray:
    """u = (2*(r >> 9) + 1) * 2^-24 in (0, 1)."""
    r = np.asarray(words, dtype=np.uint32)
    return ((r >> np.uint32(9)).astype(np.float64) * 2.0 + 1.0) * 2.0 ** -24


def gumbel_sample(x: np.ndarray, words: np.ndarray):
    """Gumbel-max token per row: argmax_v (x_v - ln(-ln u_v)), ties to the
    lower v.  Returns (tokens int32, margin = best key - second key).

    [Press] "What DiffusionGemma does": every position is evaluated at every
    step; the draw itself is the plain Gumbel-max sample of softmax(x).
    """
    u = uniform_f64(words)
    key = x - np.log(-np.log(u))
    tok = np.argmax(key, axis=1)
    top2 = -np.partition(-key, 1, axis=1)[:, :2]
    return tok.astype(np.int32), top2[:, 0] - top2[:, 1]


# --------------------------------------------------------------------------
# a7: entropy-bounded selection, a8: renoise, a9: stop
# --------------------------------------------------------------------------

def select(H: np.ndarray, bound: float = ENTROPY_BOUND, rule: int = SELECT_CUMSUM, top_k: int = 1):
    """Entropy-bounded acceptance of one canvas.

    Sort the slots by entropy (ties to the lower slot) and accept a prefix of
    that order:
      * SELECT_CUMSUM (default): with the inclusive running sum c_j, the first
        n = max(1, #{j : c_j <= bound}).  [Docs] token-selection row: the
        lowest-entropy tokens are chosen so that the bound holds; the
        cumulative-sum form is this project's reading of that
        mutual-information bound.
      * SELECT_MI: the longest prefix whose entropy sum minus its largest
        entropy is <= bound, i.e. with the exclusive running sum e_j (the sum
        over the slots ranked before j; e_0 = 0), n = #{j : e_j <= bound} >= 1.
        A bound of this shape is the usual form in the literature on
        entropy-bounded samplers; the pages do not state it.
      * SELECT_TOPK: the top_k lowest-entropy slots.
    Returns (accept uint8, n, margin) where margin is the closest call at the
    cut (for the sums: distance of the deciding sums from the bound, or the
    entropy gap at the cut; for top-k: the entropy gap at the cut).
    """
    H = np.asarray(H, dtype=np.float64)
    L = H.shape[0]
    order = np.lexsort((np.arange(L), H))
    Hs = H[order]
    c = np.cumsum(Hs)
    margins = []
    if rule == SELECT_CUMSUM:
        n = max(1, int(np.count_nonzero(c <= bound)))
        margins.append(abs(c[n - 1] - bound))
        if n < L:
            margins.append(abs(c[n] - bound))
    elif rule == SELECT_MI:
        e = np.concatenate([[0.0], c[:-1]])
        n = int(np.count_nonzero(e <= bound))
        margins.append(abs(e[n - 1] - bound))
        if n < L:
            margins.append(abs(e[n] - bound))
    elif rule == SELECT_TOPK:
        if not 1 <= top_k <= L:
            raise ValueError("top_k out of range")
        n = int(top_k)
    else:
        raise ValueError("unknown selection rule")
    acc = np.zeros(L, dtype=np.uint8)
    acc[order[:n]] = 1
    if n < L:
        margins.append(abs(Hs[n] - Hs[n - 1]))
    return acc, n, float(min(margins)) if margins else float("inf")


def renoise_tokens(b: int, k: int, L: int, V: int, seed: int) -> np.ndarray:
    """Uniform replacement tokens for canvas b at step k, int32 [L].

    [Docs] token-selection row: unselected tokens are fully renoised;
    [Report] Figure 3: the noise distribution is uniform over the vocabulary.
    Philox counter (0, slot | 1 << 16, k, b), lane 0, token = (r * V) >> 32.
    """
    k0, k1 = split_seed(seed)
    slots = np.arange(L, dtype=np.uint64)
    o = philox4x32_10(np.uint64(0), slots | np.uint64(PURPOSE_RENOISE << 16),
                      np.uint64(k), np.uint64(b), k0, k1)
    r = o[0].astype(np.uint64)
    return ((r * np.uint64(V)) >> np.uint64(32)).astype(np.int32)


def initial_canvas(b: int, block: int, L: int, V: int, seed: int) -> np.ndarray:
    """The all-noise canvas block ``block`` of canvas b starts from, int32 [L].

    [Report] Figure 4: a block is denoised from pure noise; Figure 3: the
    noise is uniform over the vocabulary.  Philox counter
    (0, slot | 3 << 16, block << 16, b), lane 0, token = (r * V) >> 32.
    """
    k0, k1 = split_seed(seed)
    slots = np.arange(L, dtype=np.uint64)
    o = philox4x32_10(np.uint64(0), slots | np.uint64(PURPOSE_INIT << 16),
                      np.uint64(counter_step(0, block)), np.uint64(b), k0, k1)
    r = o[0].astype(np.uint64)
    return ((r * np.uint64(V)) >> np.uint64(32)).astype(np.int32)


def stop_flag(H, argmax, prev_argmax, has_prev: bool, stop_entropy: float = STOP_ENTROPY):
    """Adaptive stop of one canvas.

    [Docs] adaptive-early-stopping row: stop when the canvas-mean entropy is
    below the threshold and two consecutive denoiser predictions are the
    same; the prediction is the per-slot argmax, so the first step of a
    canvas never stops.  Returns (stop, margin = |mean H - threshold|).
    """
    mean_h = float(np.mean(np.asarray(H, dtype=np.float64)))
    same = bool(np.array_equal(np.asarray(argmax), np.asarray(prev_argmax)))
    return bool(has_prev and same and mean_h < stop_entropy), abs(mean_h - stop_entropy)


# --------------------------------------------------------------------------
# one step over B canvases
# --------------------------------------------------------------------------

def denoise_step(h_bits, *, E_bits=None, q=None, s=None, B: int, L: int = 256,
                 step_idx, has_prev, prev_argmax, params: Params = Params(),
                 canvases=None, slot_chunk: int = 32):
    """One denoising step of canvases ``canvases`` (default all) of a batch.

    ``h_bits`` is [B*L, d] bf16 bits (row b*L + s is slot s of canvas b).
    ``step_idx`` [B], ``has_prev`` [B], ``prev_argmax`` [B*L].
    Returns a dict of per-slot arrays over the chosen canvases (rows in
    canvas order) and per-canvas arrays, plus the decision margins
    (``gumbel_margin``: best minus second Gumbel key; ``argmax_margin``:
    best minus second logit; ``order_margin`` and ``stop_margin`` per
    canvas, see ``select`` and ``stop_flag``).
    """
    V = (E_bits if E_bits is not None else q).shape[0]
    canvases = list(range(B)) if canvases is None else [int(c) for c in canvases]
    out = {k: [] for k in ("entropy", "sampled", "argmax", "accept", "canvas", "gumbel_margin",
                           "argmax_margin", "stop", "order_margin", "stop_margin", "n_accept")}
    for b in canvases:
        k = int(step_idx[b])
        tau = temperature(k, params.tau0, params.tau1, params.max_steps)
        z = logits(h_bits[b * L:(b + 1) * L], E_bits=E_bits, q=q, s=s)
        H = np.empty(L)
        samp = np.empty(L, dtype=np.int32)
        gm = np.empty(L)
        amax = argmax_lowest(z)
        top2 = -np.partition(-z, 1, axis=1)[:, :2]
        amargin = top2[:, 0] - top2[:, 1]
        for s0 in range(0, L, slot_chunk):
            s1 = min(L, s0 + slot_chunk)
            x = z[s0:s1] / tau
            H[s0:s1] = entropy(x)
            w = gumbel_words(np.arange(s0, s1), b, counter_step(k, params.block), V, params.seed)
            samp[s0:s1], gm[s0:s1] = gumbel_sample(x, w)
        acc, n, om = select(H, params.entropy_bound, params.selection_rule, params.top_k)
        noise = renoise_tokens(b, counter_step(k, params.block), L, V, params.seed)
        canvas = np.where(acc == 1, samp, noise).astype(np.int32)
        st, sm = stop_flag(H, amax, prev_argmax[b * L:(b + 1) * L], bool(has_prev[b]),
                           params.stop_entropy)
        for key, val in (("entropy", H), ("sampled", samp), ("argmax", amax),
                         ("accept", acc), ("canvas", canvas), ("gumbel_margin", gm),
                         ("argmax_margin", amargin)):
            out[key].append(val)
        out["stop"].append(st)
        out["order_margin"].append(om)
        out["stop_margin"].append(sm)
        out["n_accept"].append(n)
    res = {key: np.concatenate(out[key]) for key in
           ("entropy", "sampled", "argmax", "accept", "canvas", "gumbel_margin", "argmax_margin")}
    res["stop"] = np.array(out["stop"], dtype=np.int32)
    res["order_margin"] = np.array(out["order_margin"])
    res["stop_margin"] = np.array(out["stop_margin"])
    res["n_accept"] = np.array(out["n_accept"], dtype=np.int32)
    res["canvases"] = np.array(canvases, dtype=np.int32)
    return res
