"""The self-conditioning signal of a step: the expected embedding.

[Report] "DiffusionGemma Technical Report", Table 1: the model includes an
additional MLP block of 7.8M parameters for self-conditioning (about d^2
for d = 2816, i.e. one d x d projection of a d-wide signal).  The pages give
neither the signal nor the MLP.  Reading taken here: the signal of slot r is
the embedding expected under the step's tempered distribution,

    s[r] = sum_v softmax(z[r] / tau)_v E[v]      (a d-vector per slot),

a second contraction over the vocabulary against the same embedder E, in the
shape of attention with query h, keys E and values E.  The MLP that consumes
it has trained weights and is out of scope.

TEST INFRASTRUCTURE: part of the CPU oracle (see ``oracle/__init__``).
"""
from __future__ import annotations

import numpy as np

from .step import decode_bf16, decode_e4m3, logits, temperature


def expected_embedding(h_bits, *, E_bits=None, q=None, s=None, k: int, tau0: float = 0.8, tau1: float = 0.4,
                       max_steps: int = 48, v_chunk: int = 8192, abs_values: bool = False) -> np.ndarray:
    """s = softmax(z / tau_k) @ E in float64, [rows, d]; the embedder given
    as bf16 bits or as E4M3 codes q with row scales s.  Two passes over the
    vocabulary: the row maxima of x = z / tau, then the weighted sum of the
    rows of E with weights e^{x - max} and the normaliser.  With
    ``abs_values`` the weighted sum is over |E| (same weights): the scale
    sum_v p_v |E[v]| that bounds the error of a signal computed with
    rounded weights."""
    tau = temperature(k, tau0, tau1, max_steps)
    z = logits(h_bits, E_bits=E_bits, q=q, s=s)
    x = z / tau
    m = x.max(axis=1, keepdims=True)
    w = np.exp(x - m)
    V = x.shape[1]
    d = (E_bits if E_bits is not None else q).shape[1]
    out = np.zeros((x.shape[0], d), dtype=np.float64)
    for v0 in range(0, V, v_chunk):
        v1 = min(V, v0 + v_chunk)
        if E_bits is not None:
            Ec = decode_bf16(E_bits[v0:v1])
        else:
            Ec = decode_e4m3(q[v0:v1]) * np.asarray(s[v0:v1], dtype=np.float64)[:, None]
        if abs_values:
            Ec = np.abs(Ec)
        out += w[:, v0:v1] @ Ec
    return out / w.sum(axis=1, keepdims=True)
