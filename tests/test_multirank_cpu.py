"""The N > 1 host path of bench.py on CPU: two gloo ranks.

bench.py runs one replica per GPU (every sequence and KV group is independent:
no collective on the data path); the only cross-rank step is the timing
reduction (max over ranks) and rank 0 alone printing.  These tests run that
step in two spawned processes over gloo, and check that the reference arm's
other ranks exit without work.
"""
import os
import socket
import sys
from argparse import Namespace
from datetime import timedelta

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import torch
    import torch.distributed as dist

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import bench

    # rank r: times 1 + r and 5 - r: the maxima are rank 1's first, rank 0's second
    out = bench.max_over_ranks([1.0 + rank, 5.0 - rank, 0.25], world, torch.device("cpu"))
    q.put((rank, out))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    import multiprocessing as mp

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = {}
    try:
        for _ in range(2):
            r, out = q.get(timeout=120)
            got[r] = out
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    assert got[0] == got[1] == [2.0, 5.0, 0.25]


def test_max_over_ranks_single_rank_is_identity():
    torch = pytest.importorskip("torch")
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks([3.0, 1.5], 1, torch.device("cpu")) == [3.0, 1.5]


def test_reference_arm_other_ranks_do_no_work(capsys):
    sys.path.insert(0, ROOT)
    import bench

    args = Namespace(workload=1, scale=1, dense=False, topk=0, warmup=0, steps=1, gpus=2)
    bench.run_reference(args, rank=1)
    assert capsys.readouterr().out == ""
    bench.run_reference(args, rank=0)
    out = capsys.readouterr().out.strip().splitlines()
    assert len(out) == 1 and '"impl": "reference"' in out[0]
