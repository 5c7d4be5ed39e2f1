"""Helpers shared by the GPU parity tests: run the library's step on seeded
inputs and compare it with the CPU oracle under the stated tolerances.

Tolerances (from the stated parity bar):
  * logits: max |z_gpu - z_oracle| <= 1e-2 * max |z_oracle|;
  * entropy: |H_gpu - H_oracle| <= 2e-3 nats;
  * tokens, argmax, accept masks, canvas, stop: exact, except that a slot
    whose oracle decision margin is below 1e-3 may differ, for at most
    max(1, 0.1%) of the slots of a run;
  * replay: the oracle sampler fed the device's float32 logits (and its
    entropies) reproduces tokens, argmax, masks, canvas and stop bit for bit.
"""
from __future__ import annotations

import numpy as np

import oracle
import synth
from oracle.step import Params as OParams

LOGIT_REL_TOL = 1e-2
ENTROPY_TOL = 2e-3
MARGIN = 1e-3


def to_dev_bf16(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def to_dev_fp8(q, s):
    """E4M3 codes (uint8 [V, d]) and their float32 row scales on the device."""
    import torch
    return (torch.from_numpy(np.ascontiguousarray(q, dtype=np.uint8)).cuda(),
            torch.from_numpy(np.ascontiguousarray(s, dtype=np.float32)).cuda())


def run_step(h_bits, E_bits, step_idx, has_prev, prev_argmax, canvas0, params, *,
             debug=True, active=None, e_scale=None):
    """One step through the C ABI; returns numpy outputs (and logits).

    With ``e_scale`` (float32 [V]) ``E_bits`` holds E4M3 codes (uint8) and
    the FP8 head runs."""
    import torch
    import block_canvas_denoising_b200 as dg
    B = len(step_idx)
    R, d = h_bits.shape
    V = E_bits.shape[0]
    h = to_dev_bf16(h_bits)
    if e_scale is None:
        E, sc, e_dtype = to_dev_bf16(E_bits), None, dg.E_BF16
    else:
        (E, sc), e_dtype = to_dev_fp8(E_bits, e_scale), dg.E_FP8_E4M3
    dev = dict(
        canvas=torch.from_numpy(np.asarray(canvas0, np.int32).copy()).cuda(),
        prev_argmax=torch.from_numpy(np.asarray(prev_argmax, np.int32).copy()).cuda(),
        accept=torch.zeros(R, dtype=torch.uint8, device="cuda"),
        entropy=torch.zeros(R, dtype=torch.float32, device="cuda"),
        sampled=torch.zeros(R, dtype=torch.int32, device="cuda"),
        argmax=torch.zeros(R, dtype=torch.int32, device="cuda"),
        stop=torch.full((B,), -1, dtype=torch.int32, device="cuda"),
    )
    ws = dg.Workspace(B, d, V, e_dtype)
    if debug:
        logits = torch.empty((R, V), dtype=torch.float32, device="cuda")
        dg.debug_logits(h, E, step_idx, has_prev, dev["canvas"], dev["prev_argmax"], dev["accept"],
                        dev["entropy"], dev["sampled"], dev["argmax"], dev["stop"], logits, ws,
                        params, e_scale=sc, active=active)
    else:
        logits = None
        dg.denoise_step(h, E, step_idx, has_prev, dev["canvas"], dev["prev_argmax"], dev["accept"],
                        dev["entropy"], dev["sampled"], dev["argmax"], dev["stop"], ws, params,
                        e_scale=sc, active=active)
    assert dg.device_status(ws) == 0
    torch.cuda.synchronize()
    out = {k: v.cpu().numpy() for k, v in dev.items()}
    if logits is not None:
        out["logits"] = logits.cpu().numpy()
    return out


def oparams(p) -> OParams:
    return OParams(tau0=p.tau0, tau1=p.tau1, max_steps=p.max_steps, entropy_bound=p.entropy_bound,
                   stop_entropy=p.stop_entropy, seed=p.seed, selection_rule=p.selection_rule, top_k=p.top_k,
                   block=p.block)


def rows_of(canvases, L=256):
    return np.concatenate([np.arange(b * L, (b + 1) * L) for b in canvases])


def compare_with_oracle(g, h_bits, E_bits, step_idx, has_prev, prev_argmax, params, canvases=None,
                        L=256, report=None, e_scale=None):
    """Compare device outputs ``g`` with the oracle on the chosen canvases.

    With ``e_scale``, ``E_bits`` holds E4M3 codes and the oracle dequantises
    them (codes times row scale, in float64)."""
    B = len(step_idx)
    canvases = list(range(B)) if canvases is None else list(canvases)
    op = oparams(params)
    emb = dict(E_bits=E_bits) if e_scale is None else dict(q=E_bits, s=e_scale)
    ora = oracle.denoise_step(h_bits, **emb, B=B, L=L, step_idx=step_idx, has_prev=has_prev,
                              prev_argmax=prev_argmax, params=op, canvases=canvases)
    rows = rows_of(canvases, L)
    n = len(rows)
    budget = max(1, int(0.001 * n))
    mism = 0
    info = {}

    # logits (on the same rows)
    if "logits" in g:
        z_or = np.concatenate([oracle.step.logits(h_bits[b * L:(b + 1) * L], **emb)
                               for b in canvases])
        zg = g["logits"][rows].astype(np.float64)
        err = np.abs(zg - z_or).max()
        scale = np.abs(z_or).max()
        info["logit_max_abs_err"] = float(err)
        info["logit_rel_err"] = float(err / scale) if scale > 0 else (0.0 if err == 0 else float("inf"))
        assert err <= LOGIT_REL_TOL * scale, (err, scale)
        # argmax margin of the oracle's logits
        top2 = -np.partition(-z_or, 1, axis=1)[:, :2]
        amargin = top2[:, 0] - top2[:, 1]
    else:
        amargin = ora["argmax_margin"]

    # entropy
    herr = np.abs(g["entropy"][rows].astype(np.float64) - ora["entropy"]).max()
    info["entropy_max_abs_err"] = float(herr)
    assert herr <= ENTROPY_TOL, herr

    # argmax prediction
    bad = g["argmax"][rows] != ora["argmax"]
    assert np.all(amargin[bad] < MARGIN), "argmax mismatch with a clear margin"
    mism += int(bad.sum())

    # sampled tokens
    bad = g["sampled"][rows] != ora["sampled"]
    assert np.all(ora["gumbel_margin"][bad] < MARGIN), "sampled token mismatch with a clear margin"
    mism += int(bad.sum())
    info["sampled_mismatch"] = int(bad.sum())

    # accept masks / canvas / stop per canvas
    for i, b in enumerate(canvases):
        sl = slice(i * L, (i + 1) * L)
        gsl = slice(b * L, (b + 1) * L)
        macc = g["accept"][gsl] != ora["accept"][sl]
        if macc.any():
            assert ora["order_margin"][i] < MARGIN, "accept mask mismatch with a clear margin"
            mism += int(macc.sum())
        mcan = g["canvas"][gsl] != ora["canvas"][sl]
        expl = macc | (g["sampled"][gsl] != ora["sampled"][sl])
        assert not np.any(mcan & ~expl), "canvas mismatch not explained by a near-tie"
        if g["stop"][b] != ora["stop"][i]:
            assert ora["stop_margin"][i] < MARGIN, "stop flag mismatch with a clear margin"
            mism += 1
    info["mismatches"] = mism
    assert mism <= budget, (mism, budget)
    if report is not None:
        report.update(info)
    return ora, info


def check_replay(g, step_idx, has_prev, prev_argmax, params, canvases=None, L=256):
    """Bit-exact replay of the sampler on the device's logits and entropies."""
    B = len(step_idx)
    canvases = list(range(B)) if canvases is None else list(canvases)
    rows = rows_of(canvases, L)
    op = oparams(params)
    rp = oracle.replay_step(g["logits"][rows], B=B, L=L, step_idx=step_idx, has_prev=has_prev,
                            prev_argmax=prev_argmax, params=op, entropy_in=g["entropy"][rows],
                            canvases=canvases)
    assert np.array_equal(rp["sampled"], g["sampled"][rows])
    assert np.array_equal(rp["argmax"], g["argmax"][rows])
    assert np.array_equal(rp["accept"], g["accept"][rows])
    assert np.array_equal(rp["canvas"], g["canvas"][rows])
    assert np.array_equal(rp["stop"], g["stop"][canvases])
    # entropy recomputed in float64 from the device logits agrees closely
    rp64 = oracle.replay_step(g["logits"][rows], B=B, L=L, step_idx=step_idx, has_prev=has_prev,
                              prev_argmax=prev_argmax, params=op, canvases=canvases)
    herr = np.abs(rp64["entropy"] - g["entropy"][rows]).max()
    assert herr < 1e-4, herr
    return rp


def seeded_inputs(B, d, V, *, L=256, h_seed=2, e_seed=1, canvas_seed=0):
    h = synth.hidden_normal(B, L, d, seed=h_seed)
    E = synth.embedder_normal(V, d, seed=e_seed)
    canvas0 = synth.canvas_uniform(B, L, V, seed=canvas_seed)
    return h, E, canvas0
