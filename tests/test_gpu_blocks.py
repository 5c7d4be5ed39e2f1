"""Block-by-block generation through the C ABI against the oracle.

``dg_generate_blocks`` chains the adaptive loop over canvas blocks ("encode
& append": each committed block conditions the next one through the
stand-in hidden states, which take their targets from the block committed
before).  The committed blocks and the steps each canvas took must equal the
oracle's ``generate_blocks``; every block starts from ``dg_init_canvas``'
noise, which must equal the oracle's bit for bit, and draws streams of its
own.
"""
import numpy as np
import pytest

import oracle
import synth
from dg_testlib import oparams, to_dev_bf16

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import block_canvas_denoising_b200 as dg  # noqa: E402
from block_canvas_denoising_b200 import build as dg_build  # noqa: E402

dg_build.build()
L = 256


@pytest.mark.parametrize("B,V,block", [(1, 1024, 0), (3, 8192, 0), (2, 262144, 77)])
def test_init_canvas_matches_oracle(B, V, block):
    params = dg.Params(block=block, seed=99)
    c = torch.full((B * L,), -1, dtype=torch.int32, device="cuda")
    dg.init_canvas(c, B, V, params)
    torch.cuda.synchronize()
    expect = np.concatenate([oracle.step.initial_canvas(b, block, L, V, 99) for b in range(B)])
    assert np.array_equal(c.cpu().numpy(), expect)


def _gpu_blocks(E_bits, B, n_blocks, params):
    d = E_bits.shape[1]
    V = E_bits.shape[0]
    R = B * L
    E = to_dev_bf16(E_bits)
    h_buf = torch.empty((R, d), dtype=torch.bfloat16, device="cuda")
    blocks = torch.full((n_blocks, R), -1, dtype=torch.int32, device="cuda")
    canvas = torch.zeros(R, dtype=torch.int32, device="cuda")
    prev = torch.zeros(R, dtype=torch.int32, device="cuda")
    outs = dict(accept=torch.zeros(R, dtype=torch.uint8, device="cuda"),
                entropy=torch.zeros(R, dtype=torch.float32, device="cuda"),
                sampled=torch.zeros(R, dtype=torch.int32, device="cuda"),
                argmax=torch.zeros(R, dtype=torch.int32, device="cuda"),
                stop=torch.zeros(B, dtype=torch.int32, device="cuda"))
    ws = dg.Workspace(B, d, V)
    calls = []

    def hidden(j, k, canvas_t, committed_t, h_t):
        committed = committed_t.cpu().numpy()
        calls.append((j, k, committed.shape[0]))
        if k == 0:   # the block starts from its noise canvas
            expect = np.concatenate([oracle.step.initial_canvas(b, params.block + j, L, V, params.seed)
                                     for b in range(B)])
            assert np.array_equal(canvas_t.cpu().numpy(), expect)
        y = synth.block_targets(j, committed, L, V, B=B)
        h_t.copy_(to_dev_bf16(synth.loop_hidden(k, y, E_bits, seed=4 + 1000 * j)))

    steps = dg.generate_blocks(E, hidden, n_blocks, h_buf, blocks, canvas, prev, outs["accept"], outs["entropy"],
                               outs["sampled"], outs["argmax"], outs["stop"], ws, params)
    torch.cuda.synchronize()
    return blocks.cpu().numpy(), steps, calls


@pytest.mark.parametrize("B,d,V,n_blocks,block", [(2, 256, 1024, 3, 0), (1, 512, 8192, 2, 5)])
def test_generate_blocks_matches_oracle(B, d, V, n_blocks, block):
    E_bits = synth.embedder_normal(V, d, seed=1)
    params = dg.Params(block=block)
    blocks, steps, calls = _gpu_blocks(E_bits, B, n_blocks, params)

    def hidden(j, k, canvas, committed):
        y = synth.block_targets(j, committed, L, V, B=B)
        return synth.loop_hidden(k, y, E_bits, seed=4 + 1000 * j)

    ob, osteps = oracle.generate_blocks(hidden, n_blocks=n_blocks, E_bits=E_bits, B=B, L=L, params=oparams(params))
    assert np.array_equal(steps, osteps), (steps, osteps)
    assert np.array_equal(blocks, ob)
    # the callback of block j saw j committed blocks, from step 0 on
    for j in range(n_blocks):
        ks = [k for (jj, k, n) in calls if jj == j]
        assert ks == list(range(int(steps[j].max()))) and all(n == j for (jj, k, n) in calls if jj == j)
    # the blocks settle on their targets (each derived from the block before)
    for j in range(n_blocks):
        assert (blocks[j] == synth.block_targets(j, blocks, L, V, B=B)).mean() > 0.99


def test_block_streams_differ_from_the_single_block_streams():
    # one step of block 3 against the same step as block 0: other Gumbel
    # noise, so the sampled tokens of a high-entropy canvas differ
    d, V = 256, 4096
    E_bits = synth.embedder_normal(V, d, seed=1)
    h_bits = synth.hidden_normal(1, L, d, seed=2)
    from dg_testlib import run_step
    canvas0 = np.zeros(L, np.int32)
    g0 = run_step(h_bits, E_bits, [0], [0], np.zeros(L, np.int32), canvas0, dg.Params(block=0), debug=False)
    g3 = run_step(h_bits, E_bits, [0], [0], np.zeros(L, np.int32), canvas0, dg.Params(block=3), debug=False)
    assert (g0["sampled"] != g3["sampled"]).mean() > 0.9
    assert np.array_equal(g0["argmax"], g3["argmax"]) and np.array_equal(g0["entropy"], g3["entropy"])
    from dg_testlib import compare_with_oracle
    compare_with_oracle(g3, h_bits, E_bits, np.array([0], np.int32), np.zeros(1, np.uint8), np.zeros(L, np.int32),
                        dg.Params(block=3))
