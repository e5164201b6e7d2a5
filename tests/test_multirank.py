"""Two-rank plumbing of bench.py on the CPU (gloo).

`bench.py --gpus N` runs one process per GPU under torchrun: every rank runs the
whole workload, the step time is the maximum over ranks, and only rank 0 runs
and prints the reference arm.  These checks run the same helpers with two gloo
ranks on the CPU, so the N > 1 path is covered without a GPU.
"""
import multiprocessing as mp
import os
import socket
import sys
import types

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, world: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch
    import bench
    w, r, local = bench.dist_setup(None)
    dist = bench.init_group(w, "gloo")
    slowest = bench.max_over_ranks(1.5 + r, w, torch.device("cpu"))
    bench.barrier(w)
    # the reference arm: ranks other than 0 leave without work and without printing
    args = types.SimpleNamespace(steps=1, warmup=0, ref_fraction=0.01)
    rc = bench.run_reference(args, w, r) if r != 0 else None
    out.put((r, w, local, slowest, rc))
    dist.destroy_process_group()


def test_two_gloo_ranks_max_and_reference_arm():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        got = sorted(out.get(timeout=120) for _ in procs)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert [g[0] for g in got] == [0, 1]
    assert all(g[1] == 2 for g in got)
    assert [g[2] for g in got] == [0, 1]
    assert all(g[3] == pytest.approx(2.5) for g in got)   # the slowest rank's time, on every rank
    assert got[1][4] == 0                                  # rank 1: no reference work, exit status 0
    assert all(p.exitcode == 0 for p in procs)
