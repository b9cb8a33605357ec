"""The N > 1 path of bench.py on the CPU: two ranks over gloo (127.0.0.1).

Replicas share no data-path collective; the only cross-rank operations are
the timing reduction (max over ranks) and the barriers around the timed
region, which these tests exercise with real processes."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, ws: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws)
    try:
        bench.barrier(ws)
        # each replica times its own steps; the job time is the slowest one
        t = bench.max_over_ranks(10.0 + 3.5 * rank, ws)
        bench.barrier(ws)
        out.put((rank, t, bench.job_tokens_per_s(ws, 1, 524288, t)))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_job_throughput():
    ws, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, ws, port, out)) for r in range(ws)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(out.get(timeout=10) for _ in range(ws))
    # every rank sees the max (rank 1's 13.5 ms), and the whole-job value
    # counts both replicas' tokens over that time
    assert [g[1] for g in got] == [13.5, 13.5]
    assert got[0][2] == pytest.approx(2 * 524288 / 13.5e-3)


def test_single_rank_is_identity():
    assert bench.max_over_ranks(7.25, 1) == 7.25
    assert bench.job_tokens_per_s(1, 2, 1000, 4.0) == pytest.approx(2 * 1000 / 4e-3)
