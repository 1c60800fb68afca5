"""The multi-process (one rank per GPU) path of bench.py, on CPU with the gloo backend and two
ranks: per-rank batches are independent draws, the job time is the max over ranks, the
throughput counts every rank's tokens, and the reference arm works on rank 0 only."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import workloads


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [3.0, 7.5][rank]
        ms = bench.max_over_ranks(local_ms, dist)
        value = bench.job_throughput(world, 64, 10, ms)
        wl = workloads.generate("decode_bgmv", seed=bench.rank_seed("decode_bgmv", rank),
                                shapes=(("q", 64, 64, 0),))
        ids = torch.from_numpy(wl.ids.astype(np.int64))
        gathered = [torch.empty_like(ids) for _ in range(world)]
        dist.all_gather(gathered, ids)
        out.put((rank, ms, value, [g.tolist() for g in gathered]))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_time_and_draw_their_own_batches():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    for rank, ms, value, gathered in res:
        assert ms == 7.5                                  # the slowest rank sets the job time
        assert value == pytest.approx(2 * 64 * 10 / 7.5e-3)
        assert gathered[0] != gathered[1]                 # independent batches per rank
    assert res[0][3] == res[1][3]


def test_single_process_helpers():
    assert bench.max_over_ranks(4.25) == 4.25
    assert bench.job_throughput(1, 64, 1000, 8.0) == pytest.approx(8.0e6)
    assert bench.rank_seed("decode_bgmv", 1) - bench.rank_seed("decode_bgmv", 0) == 1000


def test_reference_arm_runs_on_rank_zero_only(capsys):
    class A:
        workload = "tiny_sgmv"
        steps = 1
        warmup = 3
    bench.run_reference(A(), rank=1, world=2)         # not rank 0: returns without work or output
    assert capsys.readouterr().out == ""
