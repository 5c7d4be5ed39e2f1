"""The vocabulary-sharded step on one GPU: the embedder split into S equal
shards, one dg_head_partials call per shard (as S ranks would run them),
the record blocks stacked in shard order (what the all-gather produces),
then dg_merge_partials.  The result must equal the unsharded step (tokens,
argmax, masks, canvas, stop; entropies to float32 rounding of the merge
order) and meet the oracle's parity bar, for the bf16 and the FP8 embedder.
"""
import numpy as np
import pytest

import synth
from dg_testlib import compare_with_oracle, seeded_inputs, to_dev_bf16, to_dev_fp8

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import block_canvas_denoising_b200 as dg  # noqa: E402
from block_canvas_denoising_b200 import build as dg_build  # noqa: E402

dg_build.build()
L = 256


def _outs(R, B, canvas0, prev):
    return dict(canvas=torch.from_numpy(canvas0.copy()).cuda(),
                prev_argmax=torch.from_numpy(prev.copy()).cuda(),
                accept=torch.zeros(R, dtype=torch.uint8, device="cuda"),
                entropy=torch.zeros(R, dtype=torch.float32, device="cuda"),
                sampled=torch.zeros(R, dtype=torch.int32, device="cuda"),
                argmax=torch.zeros(R, dtype=torch.int32, device="cuda"),
                stop=torch.full((B,), -1, dtype=torch.int32, device="cuda"))


def _seq(o):
    return (o["canvas"], o["prev_argmax"], o["accept"], o["entropy"], o["sampled"], o["argmax"], o["stop"])


@pytest.mark.parametrize("S,fp8", [(2, False), (4, False), (2, True)])
def test_sharded_step_equals_unsharded(S, fp8):
    B, d, V = 2, 512, 8192
    h_bits, E_bits, canvas0 = seeded_inputs(B, d, V)
    ks = np.array([7, 30], np.int32)
    hp = np.array([1, 0], np.uint8)
    prev = np.random.default_rng(3).integers(0, V, B * L).astype(np.int32)
    R = B * L
    h = to_dev_bf16(h_bits)
    params = dg.Params(seed=99)
    if fp8:
        q, s = synth.quantize_e4m3_rows(E_bits)
        E, sc = to_dev_fp8(q, s)
        et = dg.E_FP8_E4M3
    else:
        E, sc, et = to_dev_bf16(E_bits), None, dg.E_BF16

    # unsharded
    ws = dg.Workspace(B, d, V, et)
    ref = _outs(R, B, canvas0, prev)
    dg.denoise_step(h, E, ks, hp, *_seq(ref), ws, params, e_scale=sc)
    assert dg.device_status(ws) == 0
    ref = {k: v.cpu().numpy() for k, v in ref.items()}

    # sharded: S heads, stacked records, one merge
    Vs = V // S
    count = dg.partials_count(B, d, Vs, et)
    assert count > 0
    ws_s = dg.Workspace(B, d, Vs, et)
    blocks = []
    for r in range(S):
        part = torch.empty((7, R, count), dtype=torch.float32, device="cuda")
        dg.head_partials(h, E[r * Vs:(r + 1) * Vs], r * Vs, ks, part, ws_s, params,
                         e_scale=None if sc is None else sc[r * Vs:(r + 1) * Vs])
        blocks.append(part)
    stacked = torch.stack(blocks)
    out = _outs(R, B, canvas0, prev)
    dg.merge_partials(stacked, V, d, ks, hp, *_seq(out), ws_s, params)
    assert dg.device_status(ws_s) == 0
    out = {k: v.cpu().numpy() for k, v in out.items()}

    for key in ("sampled", "argmax", "accept", "canvas", "stop", "prev_argmax"):
        assert np.array_equal(out[key], ref[key]), key
    assert np.abs(out["entropy"].astype(np.float64) - ref["entropy"]).max() < 1e-5

    emb = E_bits if not fp8 else q
    compare_with_oracle(out, h_bits, emb, ks, hp, prev, params, e_scale=None if not fp8 else s)
