"""The adaptive loop run on the device (``dg_denoise_loop_graph``), and the
fault path of both loops.

One CUDA graph with a conditional (while) node runs every step: the
hidden-state graph (here a torch-captured graph that copies step k's stand-in
hidden states out of a table, reading k from the loop state), the fused head,
the merge and the loop-control kernel that commits and freezes stopped
canvases.  Its results must equal the host loop's (``dg_denoise_loop``) bit
for bit on the same hidden states -- committed canvases, steps taken, the
last step's outputs and the resume state -- and, through it, the oracle's.
"""
import numpy as np
import pytest

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


def _outs(B):
    R = B * L
    return dict(accept=torch.zeros(R, dtype=torch.uint8, device="cuda"),
                entropy=torch.zeros(R, dtype=torch.float32, device="cuda"),
                sampled=torch.zeros(R, dtype=torch.int32, device="cuda"),
                argmax=torch.zeros(R, dtype=torch.int32, device="cuda"),
                stop=torch.zeros(B, dtype=torch.int32, device="cuda"))


def _table(E_bits, y, N, k_start):
    """Stand-in hidden states of steps k_start .. N-1, [N - k_start, R*d] bf16."""
    rows = [torch.from_numpy(synth.loop_hidden(k, y, E_bits, seed=4).view(np.int16)).view(torch.bfloat16).reshape(-1)
            for k in range(k_start, N)]
    return torch.stack(rows).cuda()


def _run_graph(E, table, B, d, V, params, k_start=0, canvas0=None, prev0=None, has_prev=None, e_scale=None):
    R = B * L
    h_buf = torch.empty((R, d), dtype=torch.bfloat16, device="cuda")
    canvas = torch.from_numpy(canvas0.copy()).cuda()
    prev = torch.from_numpy(prev0.copy()).cuda()
    hp = has_prev.copy()
    outs = _outs(B)
    ws = dg.Workspace(B, d, V, dg.E_BF16 if e_scale is None else dg.E_FP8_E4M3)
    state = dg.LoopState(B)
    g = None
    if table is not None:
        g = torch.cuda.CUDAGraph(keep_graph=True)
        with torch.cuda.graph(g):
            idx = (state.k.to(torch.int64) - k_start).clamp(0, table.shape[0] - 1)
            h_buf.view(-1).copy_(torch.index_select(table, 0, idx)[0])
    steps = dg.denoise_loop_graph(E, g, h_buf, canvas, prev, hp, outs["accept"], outs["entropy"], outs["sampled"],
                                  outs["argmax"], outs["stop"], ws, state, params, k_start=k_start, e_scale=e_scale)
    torch.cuda.synchronize()
    res = {k: v.cpu().numpy() for k, v in outs.items()}
    res.update(canvas=canvas.cpu().numpy(), prev=prev.cpu().numpy(), has_prev=hp, steps=steps,
               k_after=int(state.k.item()))
    return res


def _run_host(E, table, B, d, V, params, k_start=0, canvas0=None, prev0=None, has_prev=None, e_scale=None):
    R = B * L
    h_buf = torch.empty((R, d), dtype=torch.bfloat16, device="cuda")
    canvas = torch.from_numpy(canvas0.copy()).cuda()
    prev = torch.from_numpy(prev0.copy()).cuda()
    hp = has_prev.copy()
    outs = _outs(B)
    ws = dg.Workspace(B, d, V, dg.E_BF16 if e_scale is None else dg.E_FP8_E4M3)

    def hidden(k, canvas_t, h_t):
        if table is not None:
            h_t.view(-1).copy_(table[k - k_start])

    if table is None:
        h_buf.copy_(HOLD["h"])
    steps = dg.denoise_loop(E, hidden, h_buf, canvas, prev, hp, outs["accept"], outs["entropy"], outs["sampled"],
                            outs["argmax"], outs["stop"], ws, params, k_start=k_start, e_scale=e_scale)
    torch.cuda.synchronize()
    res = {k: v.cpu().numpy() for k, v in outs.items()}
    res.update(canvas=canvas.cpu().numpy(), prev=prev.cpu().numpy(), has_prev=hp, steps=steps)
    return res


HOLD = {}


def _same(a, b):
    for key in ("canvas", "prev", "has_prev", "steps", "accept", "sampled", "argmax", "stop"):
        assert np.array_equal(a[key], b[key]), key
    assert np.array_equal(a["entropy"].view(np.uint32), b["entropy"].view(np.uint32))


@pytest.mark.parametrize("B,d,V", [(1, 256, 1024), (3, 512, 8192)])
def test_device_loop_equals_host_loop(B, d, V):
    import oracle
    E_bits = synth.embedder_normal(V, d, seed=1)
    E = to_dev_bf16(E_bits)
    y = synth.loop_targets(L, V, seed=3, B=B)
    params = dg.Params()
    table = _table(E_bits, y, params.max_steps, 0)
    kw = dict(canvas0=synth.canvas_uniform(B, L, V, seed=0), prev0=np.zeros(B * L, np.int32),
              has_prev=np.zeros(B, np.uint8))
    gd = _run_graph(E, table, B, d, V, params, **kw)
    gh = _run_host(E, table, B, d, V, params, **kw)
    _same(gd, gh)
    assert gd["k_after"] == int(gd["steps"].max())
    fin, osteps, _ = oracle.denoise_loop(lambda k, c: synth.loop_hidden(k, y, E_bits, seed=4), E_bits=E_bits, B=B,
                                         L=L, params=oparams(params), canvas=kw["canvas0"])
    assert np.array_equal(gd["steps"], osteps)
    assert (gd["canvas"] != fin).sum() <= 1


def test_device_loop_resumes_and_caps_steps():
    # resume at k = 2 with a previous prediction, and a 6-step schedule whose
    # cap is reached by the weak-signal canvas
    B, d, V = 2, 256, 1024
    E_bits = synth.embedder_normal(V, d, seed=1)
    E = to_dev_bf16(E_bits)
    y = synth.loop_targets(L, V, seed=3, B=B)
    params = dg.Params(max_steps=6, stop_entropy=1e-12)
    table = _table(E_bits, y, params.max_steps, 2)
    kw = dict(canvas0=synth.canvas_uniform(B, L, V, seed=0),
              prev0=np.random.default_rng(1).integers(0, V, B * L).astype(np.int32),
              has_prev=np.ones(B, np.uint8))
    gd = _run_graph(E, table, B, d, V, params, k_start=2, **kw)
    gh = _run_host(E, table, B, d, V, params, k_start=2, **kw)
    _same(gd, gh)
    assert np.all(gd["steps"] == 4)


def test_device_loop_without_hidden_graph_and_with_fp8():
    # no hidden-state graph: h_buf is the same every step (a settled,
    # confident state), so the loop stops at its second step
    B, d, V = 2, 256, 2048
    E_bits = synth.embedder_normal(V, d, seed=1)
    q, s = synth.quantize_e4m3_rows(E_bits)
    Eq = torch.from_numpy(q).cuda()
    sc = torch.from_numpy(s).cuda()
    y = synth.loop_targets(L, V, seed=3, B=B)
    HOLD["h"] = to_dev_bf16(synth.loop_hidden(40, y, E_bits, seed=4))
    params = dg.Params()
    kw = dict(canvas0=synth.canvas_uniform(B, L, V, seed=0), prev0=np.zeros(B * L, np.int32),
              has_prev=np.zeros(B, np.uint8))
    R = B * L
    # the graph run uses whatever h_buf holds: fill it first
    h_buf_fill = HOLD["h"]
    gd = None
    h_buf = torch.empty((R, d), dtype=torch.bfloat16, device="cuda")
    h_buf.copy_(h_buf_fill)
    canvas = torch.from_numpy(kw["canvas0"].copy()).cuda()
    prev = torch.zeros(R, dtype=torch.int32, device="cuda")
    hp = np.zeros(B, np.uint8)
    outs = _outs(B)
    ws = dg.Workspace(B, d, V, dg.E_FP8_E4M3)
    state = dg.LoopState(B)
    steps = dg.denoise_loop_graph(Eq, None, h_buf, canvas, prev, hp, outs["accept"], outs["entropy"],
                                  outs["sampled"], outs["argmax"], outs["stop"], ws, state, params, e_scale=sc)
    torch.cuda.synchronize()
    gd = {k: v.cpu().numpy() for k, v in outs.items()}
    gd.update(canvas=canvas.cpu().numpy(), prev=prev.cpu().numpy(), has_prev=hp, steps=steps)
    gh = _run_host(Eq, None, B, d, V, params, e_scale=sc, **kw)
    _same(gd, gh)
    assert np.all(gd["steps"] == 2) and (gd["canvas"] == y).mean() > 0.99


def test_device_loop_production_shape():
    d, V = 2816, 262144
    E_bits = synth.embedder_normal(V, d, seed=1)
    E = to_dev_bf16(E_bits)
    y = synth.loop_targets(L, V, seed=3)
    params = dg.Params()
    table = _table(E_bits, y, 8, 0)      # the loop stops long before step 8
    kw = dict(canvas0=synth.canvas_uniform(1, L, V, seed=0), prev0=np.zeros(L, np.int32),
              has_prev=np.zeros(1, np.uint8))
    gd = _run_graph(E, table, 1, d, V, params, **kw)
    gh = _run_host(E, table, 1, d, V, params, **kw)
    _same(gd, gh)
    assert gd["steps"][0] == 3 and (gd["canvas"] == y).mean() > 0.99


@pytest.mark.parametrize("device_loop", [False, True])
def test_loop_stops_on_a_latched_fault(device_loop):
    # the fault is made on the host: the workspace's fault word is set before
    # the loop starts (no kernel faults, traps or hangs).  Both loops run one
    # step, see the latch, stop and return the latched status; nothing was
    # committed
    B, d, V = 2, 256, 1024
    E_bits = synth.embedder_normal(V, d, seed=1)
    E = to_dev_bf16(E_bits)
    y = synth.loop_targets(L, V, seed=3, B=B)
    R = B * L
    h_buf = to_dev_bf16(synth.loop_hidden(2, y, E_bits, seed=4)).contiguous()
    canvas0 = synth.canvas_uniform(B, L, V, seed=0)
    canvas = torch.from_numpy(canvas0.copy()).cuda()
    prev = torch.zeros(R, dtype=torch.int32, device="cuda")
    hp = np.zeros(B, np.uint8)
    outs = _outs(B)
    ws = dg.Workspace(B, d, V)
    ws.buf[:4].view(torch.int32).fill_(1 << 2)      # a bounded wait that "ran out"
    torch.cuda.synchronize()
    with pytest.raises(dg.DGError) as ei:
        if device_loop:
            dg.denoise_loop_graph(E, None, h_buf, canvas, prev, hp, outs["accept"], outs["entropy"],
                                  outs["sampled"], outs["argmax"], outs["stop"], ws, dg.LoopState(B), dg.Params())
        else:
            dg.denoise_loop(E, lambda k, c, h: None, h_buf, canvas, prev, hp, outs["accept"], outs["entropy"],
                            outs["sampled"], outs["argmax"], outs["stop"], ws, dg.Params())
    assert ei.value.code == 6                         # DG_ERR_TIMEOUT
    assert dg.device_status(ws) == 0                  # reported once, then cleared
    torch.cuda.synchronize()
    # one step ran (the outputs are written) but no canvas was committed
    assert int(outs["accept"].sum()) >= B
    assert not np.array_equal(canvas.cpu().numpy(), canvas0)   # renoised by the step, not committed


def test_loop_graph_handle_runs_again_and_equals_the_one_shot_loop():
    # one handle (dg_loop_graph_create) run three times with different
    # starting canvases, first steps and previous-prediction flags; every
    # run equals the one-shot dg_denoise_loop_graph on the same inputs, bit
    # for bit.  The buffers are the handle's: each run's inputs are copied in
    B, d, V = 2, 256, 1024
    R = B * L
    E_bits = synth.embedder_normal(V, d, seed=1)
    E = to_dev_bf16(E_bits)
    y = synth.loop_targets(L, V, seed=3, B=B)
    params = dg.Params(max_steps=12)
    table = _table(E_bits, y, params.max_steps, 0)
    h_buf = torch.empty((R, d), dtype=torch.bfloat16, device="cuda")
    canvas = torch.zeros(R, dtype=torch.int32, device="cuda")
    prev = torch.zeros(R, dtype=torch.int32, device="cuda")
    outs = _outs(B)
    ws = dg.Workspace(B, d, V)
    state = dg.LoopState(B)
    g = torch.cuda.CUDAGraph(keep_graph=True)
    with torch.cuda.graph(g):
        idx = state.k.to(torch.int64).clamp(0, table.shape[0] - 1)
        h_buf.view(-1).copy_(torch.index_select(table, 0, idx)[0])
    lg = dg.LoopGraph(E, g, h_buf, canvas, prev, outs["accept"], outs["entropy"], outs["sampled"], outs["argmax"],
                      outs["stop"], ws, state, params)
    rng = np.random.default_rng(7)
    cases = [(0, np.zeros(B, np.uint8), np.zeros(R, np.int32), 0),
             (3, np.ones(B, np.uint8), rng.integers(0, V, R).astype(np.int32), 1),
             (0, np.array([1, 0], np.uint8), rng.integers(0, V, R).astype(np.int32), 2)]
    try:
        for k_start, hp0, prev0, seed in cases:
            canvas0 = synth.canvas_uniform(B, L, V, seed=seed)
            canvas.copy_(torch.from_numpy(canvas0))
            prev.copy_(torch.from_numpy(prev0))
            hp = hp0.copy()
            steps = lg.run(hp, k_start=k_start)
            torch.cuda.synchronize()
            got = {k: v.cpu().numpy() for k, v in outs.items()}
            got.update(canvas=canvas.cpu().numpy(), prev=prev.cpu().numpy(), has_prev=hp, steps=steps)
            ref_table = _table(E_bits, y, params.max_steps, k_start) if k_start else table
            ref = _run_graph(E, ref_table, B, d, V, params, k_start=k_start, canvas0=canvas0, prev0=prev0,
                             has_prev=hp0.copy())
            _same(got, ref)
            assert int(state.k.item()) == int(steps.max()) + k_start
        # a first step outside the schedule is refused before any launch
        with pytest.raises(dg.DGError) as ei:
            lg.run(np.zeros(B, np.uint8), k_start=params.max_steps)
        assert ei.value.code == 4                       # DG_ERR_RANGE
    finally:
        lg.close()
    lg.close()                                          # closing twice is harmless
