"""The N > 1 plumbing of bench.py on CPU: two gloo ranks, each with its own
replica of the decode workload (weak scaling, no data-path collective).
Checks the barrier / max-over-ranks timing and the whole-job aggregation
that the GPU run uses."""
from __future__ import annotations

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench

    rank_, world_, local = bench.dist_setup()
    try:
        assert (rank_, world_, local) == (rank, world, rank)
        bench.barrier(world)
        # each rank "measured" a different time; the job time is the slowest rank's
        ms = 10.0 + 5.0 * rank
        ms_max = bench.max_over_ranks(ms, world)
        wbytes, xbytes = bench.step_bytes()
        bytes_step = sum(wbytes + xbytes[M] for M in bench.MS)
        steps = 100
        value = world * bytes_step * steps / (ms_max * 1e-3) / 1e9
        # every rank builds its own seeded replica of the workload
        items = bench.workloads.decode125m(seed=1 + rank, M=1, layers=1)
        q.put((rank, ms_max, value, float(items[0][2].float().sum())))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_rank_weak_scaling_plumbing():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=10) for _ in range(world))
    assert [r[1] for r in res] == [15.0, 15.0]          # max over ranks, on every rank
    assert res[0][2] == pytest.approx(res[1][2])       # same whole-job value everywhere
    import bench
    wbytes, xbytes = bench.step_bytes()
    per_rank = sum(wbytes + xbytes[M] for M in bench.MS) * 100 / 15e-3 / 1e9
    assert res[0][2] == pytest.approx(2 * per_rank)    # whole job = world x per-rank work / slowest time
    assert res[0][3] != res[1][3]                      # independent replicas (different seeds)


def test_step_bytes_match_packed_format():
    import bench
    from ternary_quantized_linear_bitlinear_b200 import workloads
    wbytes, xbytes = bench.step_bytes()
    shapes = workloads.decode125m_layer_shapes()
    assert wbytes == 12 * sum(N * K for _, N, K, _ in shapes) // 4 == 18874368
    assert xbytes[8] == 8 * xbytes[1]
