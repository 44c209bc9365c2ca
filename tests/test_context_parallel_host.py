"""Host logic of sequence-sharded attention (CPU): which K/V chunks each rank
attends to, and the all-gather that assembles them, run as two gloo ranks."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from exact_softmax_attention_03_b200.context_parallel import chunk_plan


def test_chunk_plan_causal_and_full():
    assert chunk_plan(0, 4, True) == [(0, True)]
    assert chunk_plan(2, 4, True) == [(0, False), (1, False), (2, True)]
    assert chunk_plan(3, 4, False) == [(0, False), (1, False), (2, False), (3, False)]
    # every (query chunk, key chunk) pair with an allowed key is covered exactly once
    world = 5
    pairs = {(r, s) for r in range(world) for s, _ in chunk_plan(r, world, True)}
    assert pairs == {(r, s) for r in range(world) for s in range(world) if s <= r}
    with pytest.raises(ValueError):
        chunk_plan(4, 4, True)


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
        from exact_softmax_attention_03_b200.context_parallel import gather_chunks
        x = torch.full((2, 3, 1, 4), float(rank + 1))
        chunks = gather_chunks(x)
        out.put((rank, [float(c[0, 0, 0, 0]) for c in chunks], [tuple(c.shape) for c in chunks]))
    finally:
        dist.destroy_process_group()


def test_gather_chunks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, vals, shapes in res:
        assert vals == [1.0, 2.0]                    # rank order on every rank
        assert shapes == [(2, 3, 1, 4)] * 2


class _SharedPeers:
    """Stand-in for PeerKV on CPU: every rank's buffers are shared-memory
    tensors that all ranks can read, as peer memory would be."""

    def __init__(self, bufs_k, bufs_v, rank):
        self.bufs_k, self.bufs_v = bufs_k, bufs_v
        self.k, self.v = bufs_k[rank], bufs_v[rank]

    def write(self, k, v):
        self.k.copy_(k)
        self.v.copy_(v)

    def views(self, r):
        return self.bufs_k[r], self.bufs_v[r]


def _peer_worker(rank, world, port, bufs_k, bufs_v, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        from exact_softmax_attention_03_b200.context_parallel import (
            context_parallel_attention_peer)
        peers = _SharedPeers(bufs_k, bufs_v, rank)

        def attend(q, k_chunks, v_chunks, r, causal, scale):
            # what the attention step would read: the first element of every
            # chunk of its plan
            return [(s, float(k_chunks[s][0, 0, 0, 0]), float(v_chunks[s][0, 0, 0, 0]))
                    for s, _ in chunk_plan(r, len(k_chunks), causal)]

        seen = []
        shape = tuple(bufs_k[rank].shape)
        for it in range(3):                     # the buffers are reused round after round
            val = float(10 * it + rank + 1)
            seen.append(context_parallel_attention_peer(
                torch.zeros(shape), torch.full(shape, val), torch.full(shape, -val), peers,
                causal=True, attend=attend))
        out.put((rank, seen))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_peer_chunks_are_read_in_place_after_every_write(world):
    ctx = mp.get_context("spawn")
    shape = (1, 4, 2, 8)
    bufs_k = [torch.zeros(shape).share_memory_() for _ in range(world)]
    bufs_v = [torch.zeros(shape).share_memory_() for _ in range(world)]
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_peer_worker, args=(r, world, port, bufs_k, bufs_v, q))
             for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, rounds in res.items():
        for it, got in enumerate(rounds):
            want = [(s, float(10 * it + s + 1), -float(10 * it + s + 1)) for s in range(rank + 1)]
            assert got == want, (rank, it, got)


def _failing_worker(rank, world, port, bufs_k, bufs_v, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=30))
    try:
        from exact_softmax_attention_03_b200.context_parallel import (
            context_parallel_attention_peer)
        peers = _SharedPeers(bufs_k, bufs_v, rank)
        shape = tuple(bufs_k[rank].shape)

        def attend(q, k_chunks, v_chunks, r, causal, scale, fail=[True]):
            if r == 1 and fail[0]:                 # the first round fails on rank 1 only
                fail[0] = False
                raise RuntimeError("attention step failed")
            return [float(k_chunks[s][0, 0, 0, 0]) for s, _ in chunk_plan(r, len(k_chunks), causal)]

        log = []
        for it in range(2):
            val = float(10 * it + rank + 1)
            try:
                log.append(context_parallel_attention_peer(
                    torch.zeros(shape), torch.full(shape, val), torch.full(shape, -val), peers,
                    causal=True, attend=attend))
            except RuntimeError as e:
                log.append(str(e))
        out.put((rank, log))
    finally:
        dist.destroy_process_group()


def test_peer_round_error_on_one_rank_keeps_the_group_in_step():
    """A rank whose attention step raises still takes the closing barrier, so
    the next round pairs every rank's barriers correctly."""
    world, shape = 2, (1, 4, 2, 8)
    ctx = mp.get_context("spawn")
    bufs_k = [torch.zeros(shape).share_memory_() for _ in range(world)]
    bufs_v = [torch.zeros(shape).share_memory_() for _ in range(world)]
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_failing_worker, args=(r, world, port, bufs_k, bufs_v, q))
             for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[1][0] == "attention step failed"
    assert res[0][0] == [1.0]
    assert res[0][1] == [11.0] and res[1][1] == [11.0, 12.0]


def test_peer_buffers_refuse_a_chunk_that_would_broadcast():
    from exact_softmax_attention_03_b200.context_parallel import PeerKV
    peers = PeerKV.__new__(PeerKV)            # the buffers only; no rendezvous on CPU
    peers.shape, peers.dtype = (4, 8, 2, 16), torch.bfloat16
    peers.k = torch.zeros(peers.shape, dtype=peers.dtype)
    peers.v = torch.zeros(peers.shape, dtype=peers.dtype)
    small = torch.ones((1, 8, 2, 16), dtype=torch.bfloat16)     # broadcasts to the buffers
    with pytest.raises(ValueError, match="shape"):
        peers.write(small, small)
    good = torch.ones(peers.shape, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="float32"):
        peers.write(good.float(), good)
    peers.write(good, -good)
    assert float(peers.k.sum()) == good.numel() and float(peers.v.sum()) == -good.numel()
