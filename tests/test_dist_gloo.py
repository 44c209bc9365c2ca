"""The multi-GPU bench path, exercised on CPU with two gloo ranks.

Every rank runs its own independent batch (no collective in the data path);
only the timing reduction (max over ranks) crosses ranks. These tests check
that reduction, the per-rank shard seeds and the whole-job rate formula with
world_size 2 over 127.0.0.1.
"""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import attn_inputs as ai
        # per-rank "kernel times": rank r measured (1 + r) ms
        ms = 1.0 + rank
        ms_max = bench.max_over_ranks(ms, world)
        bench.barrier(world)
        q, k, v = ai.make_qkv(1, 2, 2, 8, 8, 64, seed=bench.shard_seed(rank))
        digest = float(q.float().sum())
        gathered = [None] * world
        dist.all_gather_object(gathered, (rank, ms_max, digest, bench.shard_seed(rank)))
        if rank == 0:
            out.put(gathered)
    finally:
        dist.destroy_process_group()


@pytest.fixture(scope="module")
def two_rank_results():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return sorted(res)


def test_max_over_ranks_is_the_slowest_rank(two_rank_results):
    assert [r[1] for r in two_rank_results] == [2.0, 2.0]


def test_each_rank_draws_an_independent_shard(two_rank_results):
    seeds = [r[3] for r in two_rank_results]
    digests = [r[2] for r in two_rank_results]
    assert seeds[0] != seeds[1]
    assert digests[0] != digests[1]


def test_whole_job_rate_counts_all_ranks_over_the_slowest_time():
    import bench
    # 2 ranks, 1e12 FLOP each, slowest rank 2 ms -> 1e15 FLOP/s
    assert bench.whole_job_rate(1e12, 2.0, 2) == pytest.approx(1e15)
    assert bench.whole_job_rate(5.0, 1.0, 1) == pytest.approx(5000.0)


def test_single_process_helpers_need_no_process_group():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    bench.barrier(1)
