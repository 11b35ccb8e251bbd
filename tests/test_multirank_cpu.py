"""The multi-rank benchmark logic on CPU with two gloo ranks: each rank times its own
sequence (distinct seeds, no data exchange), the reported time is the max over ranks and
the job throughput counts every rank's rows."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local = [3.0, 7.5][rank]
        m = bench.max_over_ranks(local, world, "cpu")
        m2 = bench.max_over_ranks(-local, world, "cpu")     # second collective, same order
        dist.barrier()
        q.put((rank, m, m2, bench.rank_seed(2, rank)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    out = sorted(q.get(timeout=120) for _ in ps)
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [o[1] for o in out] == [7.5, 7.5]
    assert [o[2] for o in out] == [-3.0, -3.0]
    assert out[0][3] != out[1][3]                 # independent sequences per rank
    assert bench.job_throughput(16128, 2, 7.5) == pytest.approx(2 * 16128 / 7.5e-3)


def test_single_rank_passthrough():
    assert bench.max_over_ranks(4.2, 1) == 4.2
    assert bench.job_throughput(100, 1, 1.0) == pytest.approx(1e5)
