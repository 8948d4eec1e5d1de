"""Host logic of the multi-rank (torchrun) bench path on two gloo ranks (CPU).

The data path shards by batch with no collective; the only cross-rank steps
are the barrier and the max-over-ranks reduction of the elapsed time, which
these tests exercise with the gloo backend."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    import workloads as W
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = W.BY_NAME["chunk_bf16_h2048"]
        ms_local = 10.0 + 5.0 * rank          # the slowest rank decides
        value, ms_max = bench.aggregate_throughput(ms_local, 4, wl.B * wl.T, world, device="cpu")
        bench.barrier(world)
        q.put((rank, value, ms_max, bench.rank_seed(wl, rank)))
    finally:
        dist.destroy_process_group()


def test_two_rank_aggregation_on_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    tokens = 8 * 4096
    for rank, value, ms_max, seed in res:
        assert ms_max == pytest.approx(15.0)
        assert value == pytest.approx(tokens * world * 4 / 15e-3)
    assert res[0][3] != res[1][3]           # each rank draws its own batch


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    v, ms = bench.aggregate_throughput(2.0, 10, 100, 1)
    assert ms == 2.0 and v == pytest.approx(100 * 10 / 2e-3)
