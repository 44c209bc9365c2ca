"""Sequence-sharded (context-parallel) attention over torch.distributed.

Each rank holds one equal-length chunk of the sequence: its queries and its
keys/values. The ranks all-gather the K/V chunks (NCCL over NVLink between
GPUs), each rank attends its query chunk to every chunk it may see with the
library's forward kernel, and the per-chunk results are merged with the
rescale-to-common-maximum rule ("Chapter 3: MHA Limitations, MQA, GQA, and
FlashAttention", section 3.5) by the library's merge kernel. The use is the
long-context case of "How to Reduce Attention Computation Cost in LLM
Training", section "Ring Attention and Sequence Parallelism": when one GPU's
memory is the wall, the sequence is split across NVLink-connected GPUs.

Causal masking across chunks: rank r's queries sit at global positions
[r*C, (r+1)*C); chunk s < r is wholly visible, chunk r is the usual causal
(diagonal) block, chunks s > r are wholly masked and skipped. Sliding windows
are not supported here. All arithmetic runs in the library's kernels; this
module only moves tensors and chooses calls.

Two ways to reach the other ranks' chunks: ``context_parallel_attention``
all-gathers them (NCCL), ``context_parallel_attention_peer`` lets the forward
kernel read them in place from the owners' memory (``PeerKV``), so the
transfer overlaps the products tile by tile and no gathered copy is made.
"""

from __future__ import annotations

import torch

from . import attn_fwd_f32o, attn_merge


def chunk_plan(rank: int, world: int, causal: bool):
    """``[(s, is_causal_block)]``: the K/V chunks rank ``rank`` attends to."""
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    if not causal:
        return [(s, False) for s in range(world)]
    return [(s, s == rank) for s in range(rank + 1)]


def gather_chunks(x: torch.Tensor, group=None) -> list:
    """All-gather one equal-shaped chunk per rank; returns the list in rank order."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    out = [torch.empty_like(x) for _ in range(world)]
    dist.all_gather(out, x.contiguous(), group=group)
    return out


def context_parallel_local(q, k_chunks, v_chunks, rank: int, causal: bool = True, scale=None,
                           lse=None):
    """Attention of this rank's query chunk ``q [B, C, Hq, d]`` to the gathered
    K/V chunks (``[B, C, Hkv, d]`` each, rank order). Returns ``(o, lse)``."""
    world = len(k_chunks)
    plan = chunk_plan(rank, world, causal)
    B, C, Hq, d = q.shape
    o_parts = torch.empty((len(plan), B, C, Hq, d), dtype=torch.float32, device=q.device)
    lse_parts = torch.empty((len(plan), B, Hq, C), dtype=torch.float32, device=q.device)
    for i, (s, diag) in enumerate(plan):
        attn_fwd_f32o(q, k_chunks[s], v_chunks[s], o=o_parts[i], lse=lse_parts[i], causal=diag,
                      scale=scale)
    if lse is None:
        lse = torch.empty((B, Hq, C), dtype=torch.float32, device=q.device)
    return attn_merge(o_parts, lse_parts, lse=lse)


def context_parallel_attention(q, k, v, group=None, causal: bool = True, scale=None):
    """Sequence-sharded attention: each rank passes its own chunk of Q, K, V
    (equal lengths on every rank); returns this rank's chunk of O and LSE."""
    import torch.distributed as dist
    rank = dist.get_rank(group)
    k_chunks = gather_chunks(k, group)
    v_chunks = gather_chunks(v, group)
    return context_parallel_local(q, k_chunks, v_chunks, rank, causal=causal, scale=scale)


class PeerKV:
    """K/V chunk buffers that every rank of a group can read in place.

    Each rank writes its own chunk into its buffers; ``views(r)`` returns rank
    r's buffers as tensors of this process (peer memory over NVLink for
    r != this rank). The forward kernel's tile loads then read a peer's chunk
    directly: plain TMA loads, never cluster multicast. Built on torch's
    symmetric memory; allocate once per (group, chunk shape) and reuse.
    """

    def __init__(self, shape, dtype=torch.bfloat16, device=None, group=None):
        import torch.distributed as dist
        import torch.distributed._symmetric_memory as symm
        self.group = group if group is not None else dist.group.WORLD
        self.shape, self.dtype = tuple(shape), dtype
        self.k = symm.empty(*self.shape, dtype=dtype, device=device)
        self.v = symm.empty(*self.shape, dtype=dtype, device=device)
        self._hk = symm.rendezvous(self.k, self.group)
        self._hv = symm.rendezvous(self.v, self.group)

    def write(self, k: torch.Tensor, v: torch.Tensor) -> None:
        """Copy this rank's chunk in. The chunk must match the buffers exactly:
        a copy that broadcast a smaller chunk would give every rank wrong data."""
        for t, name in ((k, "k"), (v, "v")):
            if tuple(t.shape) != self.shape:
                raise ValueError(f"{name} chunk has shape {tuple(t.shape)}, buffers hold {self.shape}")
            if t.dtype != self.dtype:
                raise ValueError(f"{name} chunk is {t.dtype}, buffers hold {self.dtype}")
            if t.device != self.k.device:
                raise ValueError(f"{name} chunk is on {t.device}, buffers are on {self.k.device}")
        self.k.copy_(k)
        self.v.copy_(v)

    def views(self, r: int):
        return (self._hk.get_buffer(r, self.shape, self.dtype),
                self._hv.get_buffer(r, self.shape, self.dtype))


def _stream_done(t: torch.Tensor) -> None:
    if t.is_cuda:
        torch.cuda.current_stream(t.device).synchronize()


def context_parallel_attention_peer(q, k, v, peers, group=None, causal: bool = True, scale=None,
                                    attend=None):
    """Sequence-sharded attention that reads the other ranks' K/V chunks in place.

    ``peers`` is this group's ``PeerKV`` for the chunk shape. Each rank writes
    its chunk into its own buffers; once every rank has (barrier), the forward
    kernel reads each visible chunk from its owner's memory; a second barrier
    holds the buffers until every rank has finished reading them. Same result
    as ``context_parallel_attention``. ``attend`` replaces the per-rank
    attention step (``context_parallel_local``'s signature), for tests.
    If the attention step raises on one rank, that rank still takes the second
    barrier before the error propagates, so the other ranks are not left
    waiting for it.
    """
    import torch.distributed as dist
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    peers.write(k, v)
    _stream_done(peers.k)
    dist.barrier(group=group)                   # every chunk written
    attend = attend or context_parallel_local
    try:
        views = [peers.views(r) for r in range(world)]
        out = attend(q, [kv[0] for kv in views], [kv[1] for kv in views], rank, causal=causal,
                     scale=scale)
        _stream_done(q)
    finally:
        dist.barrier(group=group)               # every chunk read: buffers may be rewritten
    return out
