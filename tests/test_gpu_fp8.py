"""The FP8-E4M3 embedder variant through the C ABI against the oracle.

E is quantised per vocabulary row (E4M3 codes q, float32 scale s_v =
absmax_v / 448); h stays bf16.  The oracle dequantises q * s to float64
before the head.  The device feeds the codes to E4M3 tensor-core MMAs and
splits each row of h into two E4M3 terms with a power-of-two scale
(h * 2^k_r = h1 + h2, exact for |h| >= 2^-9 max|h[r]|).
Cases: every one of the 254 finite codes in every K position with one-hot
hidden states (logits bit-exact); the split of h across its exact range and
below it; the tiny and ragged shapes of the bf16 parity suite; the
production B=1 step; a batched step with per-canvas step indices; the
adaptive loop; non-finite h reported.
"""
import numpy as np
import pytest

import oracle
import synth
from dg_testlib import (check_replay, compare_with_oracle, oparams, run_step, seeded_inputs, to_dev_bf16,
                        to_dev_fp8)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import block_canvas_denoising_b200 as dg  # noqa: E402
from block_canvas_denoising_b200 import build as dg_build  # noqa: E402

dg_build.build()
L = 256


def _fp8_case(B, d, V, ks, seeds=(2, 1, 0), has_prev=None, prev=None, params=None):
    params = params or dg.Params()
    h, E_bits, canvas0 = seeded_inputs(B, d, V, h_seed=seeds[0], e_seed=seeds[1], canvas_seed=seeds[2])
    q, s = synth.quantize_e4m3_rows(E_bits)
    hp = np.zeros(B, np.uint8) if has_prev is None else np.asarray(has_prev, np.uint8)
    prev = np.zeros(B * L, np.int32) if prev is None else prev
    ks = np.asarray(ks, np.int32)
    g = run_step(h, q, ks, hp, prev, canvas0, params, e_scale=s)
    return h, q, s, ks, hp, prev, params, g


def test_fp8_every_code_in_every_k_position_bit_exact():
    # d = 256: hidden row r is one-hot at k = r, so z[r, v] = s_v * q[v, r]
    # exactly (one non-zero product).  Row v of the codes is the cyclic
    # shift (v + k) mod 256 with the two NaN codes (0x7f, 0xff) replaced by
    # 0: every finite code -- subnormals, -0, +-448 -- meets every K
    # position, every swizzle phase and both bytes of every converted pair.
    d, V = 256, 256
    codes = (np.arange(V)[:, None] + np.arange(d)[None, :]) % 256
    codes[(codes == 0x7F) | (codes == 0xFF)] = 0
    q = codes.astype(np.uint8)
    s = (0.5 + 0.25 * (np.arange(V) % 7) * 3.0 ** -(np.arange(V) % 5)).astype(np.float32)
    h = np.zeros((L, d), np.uint16)
    h[np.arange(L), np.arange(L) % d] = 0x3F80            # bf16 1.0
    ks = np.array([0], np.int32)
    g = run_step(h, q, ks, np.zeros(1, np.uint8), np.zeros(L, np.int32),
                 synth.canvas_uniform(1, L, V, seed=0), dg.Params(), e_scale=s)
    want = (oracle.step.decode_e4m3(q) * s.astype(np.float64)[:, None]).T.astype(np.float32)  # [r, v]
    got = g["logits"] + np.float32(0.0)       # -0 -> +0 on both sides
    want = want + np.float32(0.0)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))


def test_fp8_tiny_parity_and_replay():
    h, q, s, ks, hp, prev, params, g = _fp8_case(1, 512, 8192, [0])
    report = {}
    compare_with_oracle(g, h, q, ks, hp, prev, params, report=report, e_scale=s)
    check_replay(g, ks, hp, prev, params)
    assert report["logit_rel_err"] < 1e-5


@pytest.mark.parametrize("B,d,V,ks", [
    (1, 64, 256, [5]),            # one K stage, one vocabulary tile
    (2, 192, 768, [0, 47]),       # fewer K blocks than stages, ragged split
    (3, 320, 2304, [10, 20, 30]),
    (1, 2816, 4096, [23]),        # production d
    (2, 1024, 65536, [1, 46]),    # many tiles per CTA pair
])
def test_fp8_small_shapes_parity_and_replay(B, d, V, ks):
    h, q, s, ks, hp, prev, params, g = _fp8_case(B, d, V, ks)
    compare_with_oracle(g, h, q, ks, hp, prev, params, e_scale=s)
    check_replay(g, ks, hp, prev, params)


@pytest.fixture(scope="module")
def production_fp8():
    E_bits = synth.embedder_normal(262144, 2816, seed=1)
    q, s = synth.quantize_e4m3_rows(E_bits)
    del E_bits
    return q, s


@pytest.mark.parametrize("k", [0, 47])
def test_fp8_production_single_step(production_fp8, k):
    q, s = production_fp8
    d, V = 2816, 262144
    h = synth.hidden_normal(1, L, d, seed=2)
    ks = np.array([k], np.int32)
    hp = np.zeros(1, np.uint8)
    prev = np.zeros(L, np.int32)
    params = dg.Params()
    g = run_step(h, q, ks, hp, prev, synth.canvas_uniform(1, L, V, seed=0), params, e_scale=s)
    report = {}
    compare_with_oracle(g, h, q, ks, hp, prev, params, report=report, e_scale=s)
    check_replay(g, ks, hp, prev, params)
    print(k, report)
    assert report["logit_rel_err"] < 1e-5


def test_fp8_batched_b4_per_canvas_steps(production_fp8):
    q, s = production_fp8
    B, d, V = 4, 2816, 262144
    h = synth.hidden_normal(B, L, d, seed=2)
    ks = synth.step_indices_uniform(B, 48, seed=5)
    hp = (np.arange(B) % 2).astype(np.uint8)
    prev = np.random.default_rng(6).integers(0, V, B * L).astype(np.int32)
    params = dg.Params()
    g = run_step(h, q, ks, hp, prev, synth.canvas_uniform(B, L, V, seed=0), params, e_scale=s)
    compare_with_oracle(g, h, q, ks, hp, prev, params, canvases=[3], e_scale=s)
    check_replay(g, ks, hp, prev, params, canvases=[0, 3])
    for b in range(B):
        sl = slice(b * L, (b + 1) * L)
        acc = g["accept"][sl]
        assert acc.sum() >= 1
        assert np.array_equal(g["canvas"][sl][acc == 1], g["sampled"][sl][acc == 1])
        assert np.array_equal(g["prev_argmax"][sl], g["argmax"][sl])


def _loop(q, s, E_bits, y, B, params):
    d, V = q.shape[1], q.shape[0]
    R = B * L
    Eq, sc = to_dev_fp8(q, s)
    h_buf = torch.empty((R, d), dtype=torch.bfloat16, device="cuda")
    canvas = torch.from_numpy(synth.canvas_uniform(B, L, V, seed=0)).cuda()
    prev = torch.zeros(R, dtype=torch.int32, device="cuda")
    has_prev = np.zeros(B, np.uint8)
    outs = [torch.zeros(R, dtype=torch.uint8, device="cuda"), torch.zeros(R, dtype=torch.float32, device="cuda"),
            torch.zeros(R, dtype=torch.int32, device="cuda"), torch.zeros(R, dtype=torch.int32, device="cuda"),
            torch.zeros(B, dtype=torch.int32, device="cuda")]
    ws = dg.Workspace(B, d, V, dg.E_FP8_E4M3)

    def hidden(k, canvas_t, h_t):
        h_t.copy_(to_dev_bf16(synth.loop_hidden(k, y, E_bits, seed=4)))

    steps = dg.denoise_loop(Eq, hidden, h_buf, canvas, prev, has_prev, *outs, ws, params, e_scale=sc)
    torch.cuda.synchronize()
    return canvas.cpu().numpy(), steps


@pytest.mark.parametrize("B,d,V", [(1, 256, 1024), (4, 512, 8192)])
def test_fp8_loop_matches_oracle(B, d, V):
    # the synthetic hidden states of the loop are built from the bf16 embedder
    # the codes were quantised from; the head uses the codes and scales
    E_bits = synth.embedder_normal(V, d, seed=1)
    q, s = synth.quantize_e4m3_rows(E_bits)
    y = synth.loop_targets(L, V, seed=3, B=B)
    params = dg.Params()
    canvas, steps = _loop(q, s, E_bits, y, B, params)
    fin, osteps, hist = oracle.denoise_loop(lambda k, c: synth.loop_hidden(k, y, E_bits, seed=4), q=q, s=s,
                                            B=B, L=L, params=oparams(params),
                                            canvas=synth.canvas_uniform(B, L, V, seed=0))
    for b in range(B):
        sl = slice(b * L, (b + 1) * L)
        if steps[b] != osteps[b]:
            kk = int(min(steps[b], osteps[b])) - 1
            i = hist[kk]["canvases"].index(b)
            assert abs(float(hist[kk]["mean_entropy"][i]) - params.stop_entropy) < 1e-3
        else:
            assert (canvas[sl] != fin[sl]).sum() <= 1


def test_fp8_hidden_split_exact_range():
    # Row r of h: 1.0 at k = 0 (sets the row scale 2^8) and one small value
    # h_r at k = 1 + r % 255; column 0 of the codes is 0, so
    # z[r, v] = s_v * q[v, k_r] * h_r.  The split represents h_r exactly
    # when h_r * 2^8 >= 2^-2, and then z is bit-exact; below that the split
    # is within 2^-10 * 2^-8 of h_r.
    d, V = 256, 256
    rng = np.random.default_rng(11)
    codes = rng.integers(0, 256, (V, d))
    codes[(codes & 0x7F) == 0x7F] = 0x38            # no NaN codes
    codes[:, 0] = 0
    q = codes.astype(np.uint8)
    s = (0.25 + rng.random(V)).astype(np.float32)
    expo = np.linspace(-14, -0.01, L)
    hr = synth.bf16_bits_from_f32((2.0 ** expo * np.where(np.arange(L) % 2, -1, 1)).astype(np.float32))
    h = np.zeros((L, d), np.uint16)
    h[:, 0] = 0x3F80
    kk = 1 + np.arange(L) % 255
    h[np.arange(L), kk] = hr
    g = run_step(h, q, np.array([0], np.int32), np.zeros(1, np.uint8), np.zeros(L, np.int32),
                 synth.canvas_uniform(1, L, V, seed=0), dg.Params(), e_scale=s)
    hv = synth.bf16_bits_to_f32(hr).astype(np.float64)
    qv = oracle.step.decode_e4m3(q[:, kk]).T * s.astype(np.float64)[None, :]     # [r, v]
    want = (hv[:, None] * qv).astype(np.float32) + np.float32(0.0)
    got = g["logits"] + np.float32(0.0)
    exact = np.abs(hv) * 256.0 >= 0.25
    assert exact.sum() > 100 and (~exact).sum() > 50
    assert np.array_equal(got[exact].view(np.uint32), want[exact].view(np.uint32))
    err = np.abs(got[~exact].astype(np.float64) - hv[~exact, None] * qv[~exact])
    bound = 2.0 ** -18 * np.abs(qv[~exact]) + 1e-7 * np.abs(want[~exact])
    assert np.all(err <= bound)


@pytest.mark.parametrize("val,status", [(0x4780, 0), (0xC780, 0), (0x0001, 0), (0x7F80, 9), (0xFFC0, 9)])
def test_fp8_nonfinite_hidden_is_reported(val, status):
    # +-65536 and a bf16 subnormal are fine (the row scale adapts);
    # +inf and NaN latch DG_ERR_VALUE
    B, d, V = 1, 128, 512
    h, E_bits, canvas0 = seeded_inputs(B, d, V)
    h = h.copy()
    h[7, 33] = val
    q, s = synth.quantize_e4m3_rows(E_bits)
    Eq, sc = to_dev_fp8(q, s)
    R = B * L
    ws = dg.Workspace(B, d, V, dg.E_FP8_E4M3)
    o = [torch.from_numpy(canvas0.copy()).cuda(), torch.zeros(R, dtype=torch.int32, device="cuda"),
         torch.zeros(R, dtype=torch.uint8, device="cuda"), torch.zeros(R, dtype=torch.float32, device="cuda"),
         torch.zeros(R, dtype=torch.int32, device="cuda"), torch.zeros(R, dtype=torch.int32, device="cuda"),
         torch.zeros(B, dtype=torch.int32, device="cuda")]
    dg.denoise_step(to_dev_bf16(h), Eq, [0], [0], *o, ws, dg.Params(), e_scale=sc)
    assert dg.device_status(ws) == status
    assert dg.device_status(ws) == 0          # the latch was cleared
