"""Seeded synthetic inputs shared by the tests, the bench and the oracle checks.

This module only names workload shapes and draws random numbers; it holds none
of the attention arithmetic, so both the CUDA path's callers and the oracle
checks may use it without sharing any of the method.

Recipe: one CPU ``torch.Generator`` per tensor, seeded ``seed``, ``seed + 1``,
``seed + 2`` for q, k, v; ``randn`` in float32 (iid N(0, 1)), then rounded to
bfloat16 on the host. The identical bf16 tensors go to the GPU and, upcast
exactly, to the oracle. The ``*_on`` variants draw the same way with a
generator on the given device (torch's own random numbers, none of this
library's kernels); the oracle then reads back the slices it checks.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import torch

SEED_Q = 1234


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    Nq: int
    Nk: int
    d: int
    causal: bool = True
    window_left: int = -1
    decode: bool = False          # single-query decode over a contiguous KV cache
    fp32_out: bool = False
    note: str = field(default="", compare=False)

    @property
    def scale(self) -> float:
        return 1.0 / (self.d ** 0.5)


# The five workloads the pages' scenarios translate into (tiny exact check,
# MHA causal prefill at 2K and 8K, GQA sliding window at 32K, GQA decode).
TINY = Workload("tiny exact attention B1 H2 N128 d64", 1, 2, 2, 128, 128, 64,
                causal=False, fp32_out=True)
TINY_CAUSAL = Workload("tiny exact attention B1 H2 N128 d64 causal", 1, 2, 2, 128, 128, 64,
                       causal=True, fp32_out=True)
MHA_2K = Workload("MHA causal prefill B4 H32 N2048 d128", 4, 32, 32, 2048, 2048, 128)
MHA_8K = Workload("MHA causal prefill B4 H32 N8192 d128", 4, 32, 32, 8192, 8192, 128)
GQA_SWA_32K = Workload("GQA sliding-window prefill B1 N32768 Hq32 Hkv8 d128 window_left4096",
                       1, 32, 8, 32768, 32768, 128, causal=True, window_left=4096)
GQA_DECODE = Workload("GQA decode B64 L8192 Hq32 Hkv8 d128", 64, 32, 8, 1, 8192, 128,
                      causal=True, decode=True)

ALL = [TINY, TINY_CAUSAL, MHA_2K, MHA_8K, GQA_SWA_32K, GQA_DECODE]


def _randn(shape, seed: int) -> torch.Tensor:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return torch.randn(*shape, generator=g, dtype=torch.float32).to(torch.bfloat16)


def make_qkv(B, Hq, Hkv, Nq, Nk, d, seed: int = SEED_Q):
    """bf16 CPU tensors q ``[B,Nq,Hq,d]``, k and v ``[B,Nk,Hkv,d]``."""
    q = _randn((B, Nq, Hq, d), seed)
    k = _randn((B, Nk, Hkv, d), seed + 1)
    v = _randn((B, Nk, Hkv, d), seed + 2)
    return q, k, v


def make_decode(B, Hq, Hkv, Lmax, d, seed: int = SEED_Q):
    """bf16 CPU tensors q ``[B,Hq,d]``, k_cache and v_cache ``[B,Lmax,Hkv,d]``."""
    q = _randn((B, Hq, d), seed)
    k = _randn((B, Lmax, Hkv, d), seed + 1)
    v = _randn((B, Lmax, Hkv, d), seed + 2)
    return q, k, v


def _randn_on(shape, seed: int, device) -> torch.Tensor:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return torch.randn(*shape, generator=g, dtype=torch.float32, device=device).to(torch.bfloat16)


def make_qkv_on(device, B, Hq, Hkv, Nq, Nk, d, seed: int = SEED_Q):
    """As :func:`make_qkv`, but drawn by a torch generator on ``device``: for
    tensors of several GB, which the host would take long to draw and copy.
    Same distribution (iid N(0, 1) rounded to bf16); other values."""
    q = _randn_on((B, Nq, Hq, d), seed, device)
    k = _randn_on((B, Nk, Hkv, d), seed + 1, device)
    v = _randn_on((B, Nk, Hkv, d), seed + 2, device)
    return q, k, v


def make_decode_on(device, B, Hq, Hkv, Lmax, d, seed: int = SEED_Q):
    """As :func:`make_decode`, drawn on ``device`` (see :func:`make_qkv_on`)."""
    q = _randn_on((B, Hq, d), seed, device)
    k = _randn_on((B, Lmax, Hkv, d), seed + 1, device)
    v = _randn_on((B, Lmax, Hkv, d), seed + 2, device)
    return q, k, v


def make_dout(B, Nq, Hq, d, seed: int = SEED_Q + 21):
    """bf16 CPU upstream gradient ``dO [B, Nq, Hq, d]`` (iid normal)."""
    return _randn((B, Nq, Hq, d), seed)


def make_dout_on(device, B, Nq, Hq, d, seed: int = SEED_Q + 21):
    """As :func:`make_dout`, drawn on ``device`` (see :func:`make_qkv_on`)."""
    return _randn_on((B, Nq, Hq, d), seed, device)


def make_for(w: Workload, seed: int = SEED_Q):
    if w.decode:
        return make_decode(w.B, w.Hq, w.Hkv, w.Nk, w.d, seed)
    return make_qkv(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, seed)


def varlen_lengths(n: int, lo: int, hi: int, seed: int = SEED_Q + 13) -> list:
    """``n`` sequence lengths drawn uniformly from ``[lo, hi]`` (seeded)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return [int(x) for x in torch.randint(lo, hi + 1, (n,), generator=g)]


def make_varlen(lens_q, lens_k, Hq, Hkv, d, seed: int = SEED_Q, q_offset: int = 0,
                tail: int = 0):
    """Packed bf16 CPU tensors for sequences of the given query/key lengths.

    Returns ``(q [total_q, Hq, d], k, v [total_k, Hkv, d], cu_q, cu_k)`` with
    ``cu_*`` int32 ``[B + 1]`` offsets; the first sequence starts at row
    ``q_offset`` of ``q`` and ``tail`` extra rows follow the last one (rows
    that belong to no sequence).
    """
    cu_q = [q_offset]
    for n in lens_q:
        cu_q.append(cu_q[-1] + int(n))
    cu_k = [0]
    for n in lens_k:
        cu_k.append(cu_k[-1] + int(n))
    total_q = cu_q[-1] + tail
    total_k = max(cu_k[-1], 1)
    q = _randn((total_q, Hq, d), seed)
    k = _randn((total_k, Hkv, d), seed + 1)
    v = _randn((total_k, Hkv, d), seed + 2)
    return (q, k, v, torch.tensor(cu_q, dtype=torch.int32), torch.tensor(cu_k, dtype=torch.int32))


def make_paged(k_cache, v_cache, page_size: int, seed: int = SEED_Q + 11, extra_pages: int = 3):
    """Scatter contiguous caches ``[B, Lmax, Hkv, d]`` into shuffled page pools.

    Returns ``(k_pages, v_pages, block_table)``: pools ``[num_pages, page_size,
    Hkv, d]`` (bf16, CPU) holding every ``page_size`` keys of every sequence in
    a page chosen by a seeded permutation, plus ``extra_pages`` pages of noise
    that no table entry names, and ``block_table [B, Lmax // page_size]``
    (int32) with ``block_table[b, i]`` = the page of keys
    ``[i * page_size, (i + 1) * page_size)`` of sequence ``b``. ``Lmax`` must be
    a multiple of ``page_size``.
    """
    B, Lmax, Hkv, d = k_cache.shape
    if Lmax % page_size:
        raise ValueError("Lmax must be a multiple of page_size")
    per_seq = Lmax // page_size
    num_pages = B * per_seq + extra_pages
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    perm = torch.randperm(num_pages, generator=g)[: B * per_seq]
    block_table = perm.reshape(B, per_seq).to(torch.int32).contiguous()
    k_pages = _randn((num_pages, page_size, Hkv, d), seed + 1)
    v_pages = _randn((num_pages, page_size, Hkv, d), seed + 2)
    idx = block_table.reshape(-1).long()
    k_pages[idx] = k_cache.reshape(B * per_seq, page_size, Hkv, d)
    v_pages[idx] = v_cache.reshape(B * per_seq, page_size, Hkv, d)
    return k_pages.contiguous(), v_pages.contiguous(), block_table


def ragged_seqlens(B: int, Lmax: int, seed: int = SEED_Q + 7) -> torch.Tensor:
    """int32 ``[B]`` cache lengths in ``[1, Lmax]`` (a mix of short and full rows)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    s = torch.randint(1, Lmax + 1, (B,), generator=g, dtype=torch.int32)
    s[0] = Lmax
    if B > 1:
        s[1] = 1
    return s
