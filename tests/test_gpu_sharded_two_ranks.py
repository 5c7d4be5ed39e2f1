"""The vocabulary-sharded step run by two processes: each rank computes the
head over its half of the embedder (dg_head_partials with its vocabulary
offset), the ranks all-gather their record blocks with the binding's
gather_partials over a gloo process group (through host memory), and rank 0
merges them (dg_merge_partials) and compares the result with the unsharded
step: tokens, argmax, accept mask, canvas and stop exactly, entropies to the
float32 rounding of the merge order.

Both ranks share the one GPU of this machine; their kernels never wait on
one another (the exchange is a host-side collective between launches).
"""
import os
import socket

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

B, D, V, L = 2, 512, 8192, 256


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_path):
    import sys
    import datetime
    import torch.distributed as dist
    here = os.path.dirname(os.path.abspath(__file__))
    sys.path.insert(0, here)
    sys.path.insert(0, os.path.dirname(here))
    import block_canvas_denoising_b200 as dg
    from dg_testlib import seeded_inputs, to_dev_bf16

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(0)
    h_bits, E_bits, canvas0 = seeded_inputs(B, D, V)
    ks = np.array([7, 30], np.int32)
    hp = np.array([1, 0], np.uint8)
    prev = np.random.default_rng(3).integers(0, V, B * L).astype(np.int32)
    R = B * L
    h = to_dev_bf16(h_bits)
    E = to_dev_bf16(E_bits)
    params = dg.Params(seed=99)
    Vs = V // world
    count = dg.partials_count(B, D, Vs, dg.E_BF16)
    ws_s = dg.Workspace(B, D, Vs)
    part = torch.empty((7, R, count), dtype=torch.float32, device="cuda")
    dg.head_partials(h, E[rank * Vs:(rank + 1) * Vs], rank * Vs, [int(k) for k in ks], part, ws_s, params)
    torch.cuda.synchronize()
    assert dg.device_status(ws_s) == 0
    gathered = dg.gather_partials(part.cpu())          # [world, 7, R, count], host memory (gloo)
    if rank == 0:
        def outs():
            return (torch.from_numpy(canvas0.copy()).cuda(), torch.from_numpy(prev.copy()).cuda(),
                    torch.zeros(R, dtype=torch.uint8, device="cuda"),
                    torch.zeros(R, dtype=torch.float32, device="cuda"),
                    torch.zeros(R, dtype=torch.int32, device="cuda"),
                    torch.zeros(R, dtype=torch.int32, device="cuda"),
                    torch.full((B,), -1, dtype=torch.int32, device="cuda"))
        o = outs()
        dg.merge_partials(gathered.cuda(), V, D, [int(k) for k in ks], hp, *o, ws_s, params)
        ws = dg.Workspace(B, D, V)
        r = outs()
        dg.denoise_step(h, E, [int(k) for k in ks], hp, *r, ws, params)
        torch.cuda.synchronize()
        assert dg.device_status(ws) == 0 and dg.device_status(ws_s) == 0
        names = ("canvas", "prev_argmax", "accept", "entropy", "sampled", "argmax", "stop")
        np.savez(out_path, **{"sh_" + n: t.cpu().numpy() for n, t in zip(names, o)},
                 **{"un_" + n: t.cpu().numpy() for n, t in zip(names, r)})
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_sharded_step_equals_unsharded(tmp_path):
    import torch.multiprocessing as mp
    out_path = str(tmp_path / "res.npz")
    mp.spawn(_rank_main, args=(2, _free_port(), out_path), nprocs=2, join=True)
    res = np.load(out_path)
    for n in ("canvas", "prev_argmax", "accept", "sampled", "argmax", "stop"):
        assert np.array_equal(res["sh_" + n], res["un_" + n]), n
    assert np.abs(res["sh_entropy"].astype(np.float64) - res["un_entropy"]).max() < 1e-5
