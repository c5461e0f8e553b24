"""The benchmark's multi-rank host logic on CPU: two `gloo` ranks (replicas only, no data exchange).

The GPU path runs one replica per GPU and combines the ranks' device-timed durations by taking the
slowest rank; the reference arm runs on rank 0 alone.  Both are checked here without a GPU.
"""
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        # rank r's step took 1 + r ms and its second figure 5 - r ms: each maximum is another rank's
        out = bench.max_over_ranks([1.0 + rank, 5.0 - rank], torch.device("cpu"), world)
        q.put((rank, out))
    finally:
        torch.distributed.destroy_process_group()


def test_max_over_ranks_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        got = sorted(q.get(timeout=120) for _ in procs)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert got == [(0, [2.0, 5.0]), (1, [2.0, 5.0])]
    assert all(p.exitcode == 0 for p in procs)


def test_max_over_ranks_single_rank_is_identity():
    assert bench.max_over_ranks([3, 4.5], None, 1) == [3.0, 4.5]


def test_reference_arm_runs_on_rank_zero_only():
    class Args:
        config, steps, warmup = "tiny", 1, 1
    assert bench.run_reference(Args(), rank=1, world=2) is None
