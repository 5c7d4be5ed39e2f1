"""Multi-rank plumbing of the bench on CPU (gloo, world size 2).

The step partitions by canvas: every rank runs its own canvases on its own
GPU and the only cross-rank traffic is the barrier and the max over ranks of
the timings.  These tests run that host-side logic with two gloo ranks.
"""
import os
import socket
import subprocess
import sys
from datetime import timedelta

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                           world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench
        got = bench.reduce_max([float(rank), 10.0 - rank, 3.5], dist)
        q.put((rank, got, bench.rank_seeds(rank)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_per_rank_inputs_on_gloo():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    out.sort()
    for rank, got, _ in out:
        assert got == [1.0, 10.0, 3.5], (rank, got)
    seeds = [s for _, _, s in out]
    assert seeds[0] != seeds[1]                      # each rank its own canvas and stream
    assert seeds[0][0] != seeds[1][0] and seeds[0][1] != seeds[1][1]


def test_reduce_max_alone_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max([2.0, 5.0], None) == [2.0, 5.0]


def test_reference_arm_on_nonzero_rank_exits_quietly():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "0"],
                       env=env, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-500:]
    assert r.stdout.strip() == ""


def _gather_worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                           world_size=world, timeout=timedelta(seconds=60))
    try:
        import block_canvas_denoising_b200 as dg
        local = torch.arange(7 * 4 * 3, dtype=torch.float32).view(7, 4, 3) + 1000.0 * rank
        out = dg.gather_partials(local)
        q.put((rank, tuple(out.shape), out[:, 2, 1, 0].tolist(), bool(torch.equal(out[rank], local))))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_vocab_sharded_records_gathered_in_rank_order_on_gloo():
    # the sharded step's only collective: every rank ends with all ranks'
    # record blocks, rank r's at index r (the merge's shard order)
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_gather_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    v = 2 * 12 + 1 * 3 + 0
    for rank, shape, vals, own in out:
        assert shape == (2, 7, 4, 3) and own
        assert vals == [float(v), 1000.0 + v]
