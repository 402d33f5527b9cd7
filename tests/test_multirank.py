"""The multi-rank host logic of bench.py on CPU: two gloo ranks.

Each rank runs its own batch of heads (weak scaling, no data-path exchange);
the only collectives are the timing barrier and reductions of per-rank numbers
(the max of the step times, the sum of the computed work).  The reference arm
runs on rank 0 only.
"""

import contextlib
import io
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, results):
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        import bench
        from workloads import WORKLOADS, make_qkv

        w = bench.rank_workload(WORKLOADS["tiny_s256"], rank)
        q, _, _ = make_qkv(w, device="cpu")
        # every rank's inputs differ (its own heads), shapes agree
        sums = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(sums, torch.tensor([float(q.double().abs().sum())], dtype=torch.float64))
        distinct = len({round(float(x), 6) for x in sums}) == world
        shapes = [None] * world
        dist.all_gather_object(shapes, tuple(q.shape))
        ms_max = bench.reduce_over_ranks(10.0 + rank, "max", True, "cpu")
        work = bench.reduce_over_ranks(1.5 * (rank + 1), "sum", True, "cpu")
        dist.barrier()
        # the reference arm: rank 0 prints one line, the other ranks do nothing
        out = io.StringIO()
        if rank != 0:
            with contextlib.redirect_stdout(out):
                os.environ["RANK"] = str(rank)
                bench.run_reference(type("A", (), {"gpus": world, "steps": 1, "warmup": 1})(), WORKLOADS["tiny_s256"])
        results[rank] = (distinct, len(set(shapes)) == 1, ms_max, work, out.getvalue())
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_weak_scaling_logic():
    world = 2
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    results = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    for p in procs:
        if p.is_alive():
            p.kill()
            pytest.fail("a rank did not finish")
        assert p.exitcode == 0
    for r in range(world):
        distinct, same_shape, ms_max, work, ref_out = results[r]
        assert distinct and same_shape
        assert ms_max == 11.0            # the slowest rank's time
        assert work == 1.5 + 3.0         # every rank's work
    assert results[1][4] == ""           # rank 1 runs no reference work
