"""Pins for block-by-block generation in the oracle (encode & append).

Block 0 is the plain adaptive loop from the block's noise canvas; every
block draws streams of its own (Gumbel noise, renoise, starting canvas),
distinct from every other block's; the hidden-state producer of block j
sees exactly the blocks committed before it; the starting canvas is uniform.
"""
import numpy as np
from scipy import stats

import synth
from oracle import denoise_loop, generate_blocks, step as S
from oracle.step import Params

L, d, V, B = 256, 256, 1024, 2


def _stand_in(E):
    seen = []

    def hidden(j, k, canvas, committed):
        seen.append((j, k, committed.copy()))
        y = synth.block_targets(j, committed, L, V, B=B)
        return synth.loop_hidden(k, y, E, seed=4 + 1000 * j)
    return hidden, seen


def test_counter_step_word():
    assert S.counter_step(5, 0) == 5 and S.counter_step(5, 3) == 5 + (3 << 16)
    for bad in ((1 << 16, 0), (0, 1 << 16), (-1, 0)):
        try:
            S.counter_step(*bad)
        except ValueError:
            continue
        raise AssertionError(bad)


def test_block_zero_is_the_plain_loop_from_its_noise_canvas():
    E = synth.embedder_normal(V, d, seed=1)
    hidden, _ = _stand_in(E)
    blocks, steps = generate_blocks(hidden, n_blocks=1, E_bits=E, B=B, L=L)
    canvas0 = np.concatenate([S.initial_canvas(b, 0, L, V, 1234) for b in range(B)])
    y = synth.block_targets(0, None, L, V, B=B)
    fin, st, _ = denoise_loop(lambda k, c: synth.loop_hidden(k, y, E, seed=4), E_bits=E, B=B, L=L,
                              canvas=canvas0)
    assert np.array_equal(blocks[0], fin) and np.array_equal(steps[0], st)


def test_blocks_see_the_committed_prefix_and_depend_on_it():
    E = synth.embedder_normal(V, d, seed=1)
    hidden, seen = _stand_in(E)
    blocks, steps = generate_blocks(hidden, n_blocks=3, E_bits=E, B=B, L=L)
    assert np.all(steps >= 2) and np.all(steps < 48)
    for j, k, committed in seen:
        assert committed.shape == (j, B * L)
        assert np.array_equal(committed, blocks[:j])
    # every block settles on its targets, which follow from the block before
    for j in range(3):
        y = synth.block_targets(j, blocks, L, V, B=B)
        assert (blocks[j] == y).mean() > 0.99
    assert not np.array_equal(blocks[1], blocks[2])


def test_every_block_draws_its_own_streams():
    seed = 1234
    w0 = S.gumbel_words(np.arange(4), 0, S.counter_step(3, 0), 64, seed)
    w1 = S.gumbel_words(np.arange(4), 0, S.counter_step(3, 1), 64, seed)
    assert not np.any(w0 == w1)
    r0 = S.renoise_tokens(0, S.counter_step(3, 0), L, V, seed)
    r1 = S.renoise_tokens(0, S.counter_step(3, 1), L, V, seed)
    assert (r0 == r1).mean() < 0.02
    c0 = S.initial_canvas(0, 0, L, V, seed)
    c1 = S.initial_canvas(0, 1, L, V, seed)
    assert (c0 == c1).mean() < 0.02
    # the starting canvas is not a renoise draw of any step of the block
    assert (c0 != S.renoise_tokens(0, S.counter_step(0, 0), L, V, seed)).mean() > 0.98


def test_initial_canvas_is_uniform():
    # 64 canvases x 256 slots over V = 64 tokens: chi-square against uniform
    Vs = 64
    toks = np.concatenate([S.initial_canvas(b, j, L, Vs, 99) for b in range(8) for j in range(8)])
    counts = np.bincount(toks, minlength=Vs)
    assert stats.chisquare(counts).pvalue > 1e-4
