"""Exact softmax attention for B200 (sm_100a): Python binding of libattn.so.

The functions here carry the C ABI's names (include/attn.h) and only marshal
torch tensors into pointers, sizes and the current CUDA stream; every step of
the computation runs in the library's kernels. There is no CPU path: a tensor
that is not a contiguous CUDA tensor of the right dtype is rejected, and a
missing library raises.

Layouts: q, o ``[B, Nq, Hq, d]``; k, v ``[B, Nk, Hkv, d]`` (bf16); lse
``[B, Hq, Nq]`` float32. Decode: q, o ``[B, Hq, d]``; caches
``[B, Lmax, Hkv, d]``; lse ``[B, Hq]``.
"""

from __future__ import annotations

import math

import torch

from ._lib import AttnError, check, load  # noqa: F401

__all__ = ["attn_fwd", "attn_fwd_f32o", "attn_fwd_varlen", "attn_bwd", "attn_bwd_workspace_bytes",
           "attn_merge", "attn_decode", "attn_decode_paged",
           "attn_decode_workspace_bytes", "attn_decode_noalloc",
           "attn_device_status", "attn_last_error", "attn_launch_count", "AttnError"]


def _stream_handle(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _need(t: torch.Tensor, name: str, dtype, ndim: int):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (no CPU path)")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _shape(t: torch.Tensor, name: str, shape):
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _same_device(ref: torch.Tensor, *named):
    """Every operand on the device of ``ref`` (the kernels read them all there)."""
    for t, name in named:
        if t is not None and t.device != ref.device:
            raise ValueError(f"{name} is on {t.device}, expected {ref.device}")


def _fwd(q, k, v, o, lse, causal, window_left, scale, stream, f32o):
    _need(q, "q", torch.bfloat16, 4)
    _need(k, "k", torch.bfloat16, 4)
    _need(v, "v", torch.bfloat16, 4)
    B, Nq, Hq, d = q.shape
    _, Nk, Hkv, _ = k.shape
    if k.shape[0] != B or k.shape[3] != d or v.shape != k.shape:
        raise ValueError("k, v must be [B, Nk, Hkv, d] matching q")
    out_dtype = torch.float32 if f32o else torch.bfloat16
    if o is None:
        o = torch.empty((B, Nq, Hq, d), dtype=out_dtype, device=q.device)
    _need(o, "o", out_dtype, 4)
    if tuple(o.shape) != (B, Nq, Hq, d):
        raise ValueError("o must be [B, Nq, Hq, d]")
    if lse is not None:
        _need(lse, "lse", torch.float32, 3)
        if tuple(lse.shape) != (B, Hq, Nq):
            raise ValueError("lse must be [B, Hq, Nq]")
    _same_device(q, (k, "k"), (v, "v"), (o, "o"), (lse, "lse"))
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    fn = load().attn_fwd_f32o if f32o else load().attn_fwd
    check(fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
             lse.data_ptr() if lse is not None else None,
             B, Hq, Hkv, Nq, Nk, d, float(scale), int(bool(causal)),
             int(window_left), _stream_handle(stream)))
    return o, lse


def attn_fwd(q, k, v, o=None, lse=None, causal=False, window_left=-1, scale=None, stream=None):
    """Forward attention, bf16 output. Returns ``(o, lse)`` (lse as passed, may be None)."""
    return _fwd(q, k, v, o, lse, causal, window_left, scale, stream, False)


def attn_fwd_f32o(q, k, v, o=None, lse=None, causal=False, window_left=-1, scale=None, stream=None):
    """Forward attention, float32 output. Returns ``(o, lse)``."""
    return _fwd(q, k, v, o, lse, causal, window_left, scale, stream, True)


def attn_fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, o=None,
                    lse=None, causal=False, window_left=-1, scale=None, stream=None):
    """Forward attention over packed variable-length sequences. Returns ``(o, lse)``.

    ``q [total_q, Hq, d]``, ``k``/``v [total_k, Hkv, d]`` (bf16, CUDA);
    ``cu_seqlens_q``/``cu_seqlens_k`` int32 ``[B + 1]`` on the device (sequence
    ``b`` owns rows ``[cu[b], cu[b+1])``); ``max_seqlen_q``/``max_seqlen_k`` are
    host ints bounding every sequence's length. ``lse`` is ``[Hq, total_q]``.
    """
    _need(q, "q", torch.bfloat16, 3)
    _need(k, "k", torch.bfloat16, 3)
    _need(v, "v", torch.bfloat16, 3)
    _need(cu_seqlens_q, "cu_seqlens_q", torch.int32, 1)
    _need(cu_seqlens_k, "cu_seqlens_k", torch.int32, 1)
    total_q, Hq, d = q.shape
    total_k, Hkv, dk = k.shape
    if dk != d or v.shape != k.shape:
        raise ValueError("k and v must be [total_k, Hkv, d] matching q")
    B = cu_seqlens_q.shape[0] - 1
    if B < 1 or cu_seqlens_k.shape[0] != B + 1:
        raise ValueError("cu_seqlens_q and cu_seqlens_k must both have B + 1 entries")
    if o is None:
        o = torch.empty((total_q, Hq, d), dtype=torch.bfloat16, device=q.device)
    _need(o, "o", torch.bfloat16, 3)
    _shape(o, "o", (total_q, Hq, d))
    if lse is not None:
        _need(lse, "lse", torch.float32, 2)
        _shape(lse, "lse", (Hq, total_q))
    _same_device(q, (k, "k"), (v, "v"), (cu_seqlens_q, "cu_seqlens_q"),
                 (cu_seqlens_k, "cu_seqlens_k"), (o, "o"), (lse, "lse"))
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    check(load().attn_fwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                 lse.data_ptr() if lse is not None else None,
                                 cu_seqlens_q.data_ptr(), cu_seqlens_k.data_ptr(), B, Hq, Hkv,
                                 total_q, total_k, int(max_seqlen_q), int(max_seqlen_k), d,
                                 float(scale), int(bool(causal)), int(window_left),
                                 _stream_handle(stream)))
    return o, lse


def attn_bwd_workspace_bytes(B: int, Hq: int, Nq: int, d: int) -> int:
    return int(load().attn_bwd_workspace_bytes(B, Hq, Nq, d))


def attn_bwd(q, k, v, o, lse, dout, causal=False, window_left=-1, scale=None, dq=None, dk=None,
             dv=None, workspace=None, stream=None):
    """Gradients of :func:`attn_fwd`. Returns ``(dq, dk, dv)`` (bf16).

    ``o`` and ``lse`` are what ``attn_fwd`` returned for the same inputs and
    mask; ``dout`` is the upstream gradient, shaped like ``o``. ``workspace``
    (``attn_bwd_workspace_bytes(...)`` bytes) is allocated here if not given.
    """
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (dout, "dout")):
        _need(t, n, torch.bfloat16, 4)
    _need(lse, "lse", torch.float32, 3)
    B, Nq, Hq, d = q.shape
    _, Nk, Hkv, _ = k.shape
    if o.shape != q.shape or dout.shape != q.shape or v.shape != k.shape:
        raise ValueError("o and dout must be shaped like q, v like k")
    if k.shape[0] != B or k.shape[3] != d:
        raise ValueError("k, v must be [B, Nk, Hkv, d] matching q")
    _shape(lse, "lse", (B, Hq, Nq))
    for t, n, like in ((dq, "dq", q), (dk, "dk", k), (dv, "dv", v)):
        if t is not None:
            _need(t, n, torch.bfloat16, 4)
            _shape(t, n, like.shape)
    if workspace is not None and not isinstance(workspace, torch.Tensor):
        raise TypeError("workspace must be a torch.Tensor")
    _same_device(q, (k, "k"), (v, "v"), (o, "o"), (lse, "lse"), (dout, "dout"), (dq, "dq"),
                 (dk, "dk"), (dv, "dv"), (workspace, "workspace"))
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    need = attn_bwd_workspace_bytes(B, Hq, Nq, d)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    check(load().attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), dout.data_ptr(),
                          lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, Hq, Hkv,
                          Nq, Nk, d, float(scale), int(bool(causal)), int(window_left),
                          workspace.data_ptr(), ws_bytes, _stream_handle(stream)))
    return dq, dk, dv


def attn_merge(o_parts, lse_parts, o=None, lse=None, stream=None):
    """Merge per-key-shard results. ``o_parts [R, B, Nq, Hq, d]`` f32 and
    ``lse_parts [R, B, Hq, Nq]`` f32 (CUDA). Returns ``(o bf16 [B, Nq, Hq, d], lse)``."""
    _need(o_parts, "o_parts", torch.float32, 5)
    _need(lse_parts, "lse_parts", torch.float32, 4)
    R, B, Nq, Hq, d = o_parts.shape
    if tuple(lse_parts.shape) != (R, B, Hq, Nq):
        raise ValueError("lse_parts must be [R, B, Hq, Nq] matching o_parts")
    if o is None:
        o = torch.empty((B, Nq, Hq, d), dtype=torch.bfloat16, device=o_parts.device)
    _need(o, "o", torch.bfloat16, 4)
    _shape(o, "o", (B, Nq, Hq, d))
    if lse is not None:
        _need(lse, "lse", torch.float32, 3)
        _shape(lse, "lse", (B, Hq, Nq))
    _same_device(o_parts, (lse_parts, "lse_parts"), (o, "o"), (lse, "lse"))
    check(load().attn_merge(o_parts.data_ptr(), lse_parts.data_ptr(), R, o.data_ptr(),
                            lse.data_ptr() if lse is not None else None, B, Nq, Hq, d,
                            _stream_handle(stream)))
    return o, lse


def attn_decode_workspace_bytes(B: int, Hq: int, d: int, num_splits: int = 0, Lmax: int = 1) -> int:
    return int(load().attn_decode_workspace_bytes(B, Hq, d, num_splits, Lmax))


def attn_decode(q, k_cache, v_cache, o=None, lse=None, seqlens=None, window_left=-1,
                scale=None, num_splits=0, workspace=None, stream=None):
    """Single-query decode over a contiguous KV cache. Returns ``(o, lse)``.

    ``workspace`` is a caller-owned CUDA buffer of at least
    ``attn_decode_workspace_bytes(...)`` bytes; if None, one is allocated here
    with torch (the library itself never allocates).
    """
    _need(q, "q", torch.bfloat16, 3)
    _need(k_cache, "k_cache", torch.bfloat16, 4)
    _need(v_cache, "v_cache", torch.bfloat16, 4)
    B, Hq, d = q.shape
    _, Lmax, Hkv, _ = k_cache.shape
    if k_cache.shape[0] != B or k_cache.shape[3] != d or v_cache.shape != k_cache.shape:
        raise ValueError("caches must be [B, Lmax, Hkv, d] matching q")
    if o is None:
        o = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=q.device)
    _need(o, "o", torch.bfloat16, 3)
    _shape(o, "o", (B, Hq, d))
    if lse is not None:
        _need(lse, "lse", torch.float32, 2)
        _shape(lse, "lse", (B, Hq))
    if seqlens is not None:
        _need(seqlens, "seqlens", torch.int32, 1)
        _shape(seqlens, "seqlens", (B,))
    _same_device(q, (k_cache, "k_cache"), (v_cache, "v_cache"), (o, "o"), (lse, "lse"),
                 (seqlens, "seqlens"), (workspace, "workspace"))
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    need = attn_decode_workspace_bytes(B, Hq, d, num_splits, Lmax)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    if not isinstance(workspace, torch.Tensor) or not workspace.is_cuda:
        raise ValueError("workspace must be a CUDA tensor")
    ws_bytes = workspace.numel() * workspace.element_size()
    check(load().attn_decode(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), o.data_ptr(),
                             lse.data_ptr() if lse is not None else None,
                             seqlens.data_ptr() if seqlens is not None else None,
                             B, Hq, Hkv, Lmax, d, float(scale), int(window_left), int(num_splits),
                             workspace.data_ptr(), ws_bytes, _stream_handle(stream)))
    return o, lse


def attn_decode_paged(q, k_pages, v_pages, block_table, o=None, lse=None, seqlens=None,
                      window_left=-1, scale=None, num_splits=0, workspace=None, stream=None):
    """Single-query decode over a paged KV cache. Returns ``(o, lse)``.

    ``k_pages``/``v_pages`` are ``[num_pages, page_size, Hkv, d]`` bf16 pools;
    ``block_table`` is ``[B, pages_per_seq]`` int32 on the device: logical key
    ``t`` of sequence ``b`` lives at row ``t % page_size`` of page
    ``block_table[b, t // page_size]``. Everything else is as in
    :func:`attn_decode` with ``Lmax = pages_per_seq * page_size``.
    """
    _need(q, "q", torch.bfloat16, 3)
    _need(k_pages, "k_pages", torch.bfloat16, 4)
    _need(v_pages, "v_pages", torch.bfloat16, 4)
    _need(block_table, "block_table", torch.int32, 2)
    B, Hq, d = q.shape
    num_pages, page_size, Hkv, _ = k_pages.shape
    if k_pages.shape[3] != d or v_pages.shape != k_pages.shape:
        raise ValueError("page pools must be [num_pages, page_size, Hkv, d] matching q")
    if block_table.shape[0] != B:
        raise ValueError("block_table must be [B, pages_per_seq]")
    pages_per_seq = block_table.shape[1]
    if o is None:
        o = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=q.device)
    _need(o, "o", torch.bfloat16, 3)
    _shape(o, "o", (B, Hq, d))
    if lse is not None:
        _need(lse, "lse", torch.float32, 2)
        _shape(lse, "lse", (B, Hq))
    if seqlens is not None:
        _need(seqlens, "seqlens", torch.int32, 1)
        _shape(seqlens, "seqlens", (B,))
    _same_device(q, (k_pages, "k_pages"), (v_pages, "v_pages"), (block_table, "block_table"),
                 (o, "o"), (lse, "lse"), (seqlens, "seqlens"), (workspace, "workspace"))
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    need = attn_decode_workspace_bytes(B, Hq, d, num_splits, pages_per_seq * page_size)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    if not isinstance(workspace, torch.Tensor) or not workspace.is_cuda:
        raise ValueError("workspace must be a CUDA tensor")
    ws_bytes = workspace.numel() * workspace.element_size()
    check(load().attn_decode_paged(q.data_ptr(), k_pages.data_ptr(), v_pages.data_ptr(), o.data_ptr(),
                                   lse.data_ptr() if lse is not None else None,
                                   block_table.data_ptr(),
                                   seqlens.data_ptr() if seqlens is not None else None,
                                   B, Hq, Hkv, num_pages, page_size, pages_per_seq, d, float(scale),
                                   int(window_left), int(num_splits), workspace.data_ptr(), ws_bytes,
                                   _stream_handle(stream)))
    return o, lse


def attn_decode_noalloc(q, k_cache, v_cache, o=None, lse=None, seqlens=None, window_left=-1,
                        scale=None, num_splits=0, stream=None):
    """Decode like :func:`attn_decode`, but the library keeps the partial results
    in its own fixed device scratch, so no workspace is passed or allocated.

    For callers that must not allocate device memory themselves (their host
    program owns all device memory through its own pool, or an allocation's
    possible device synchronisation is not acceptable on their path). ``o``
    (and ``lse``, if wanted) must still be given, or ``o`` is allocated here by
    torch for convenience. Calls on one device share the scratch: do not let
    two of them overlap on the GPU. Sizes needing more than
    ``ATTN_DECODE_NOALLOC_SCRATCH_BYTES`` of partials raise ``AttnError``.
    """
    _need(q, "q", torch.bfloat16, 3)
    _need(k_cache, "k_cache", torch.bfloat16, 4)
    _need(v_cache, "v_cache", torch.bfloat16, 4)
    B, Hq, d = q.shape
    _, Lmax, Hkv, _ = k_cache.shape
    if k_cache.shape[0] != B or k_cache.shape[3] != d or v_cache.shape != k_cache.shape:
        raise ValueError("caches must be [B, Lmax, Hkv, d] matching q")
    if o is None:
        o = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=q.device)
    _need(o, "o", torch.bfloat16, 3)
    _shape(o, "o", (B, Hq, d))
    if lse is not None:
        _need(lse, "lse", torch.float32, 2)
        _shape(lse, "lse", (B, Hq))
    if seqlens is not None:
        _need(seqlens, "seqlens", torch.int32, 1)
        _shape(seqlens, "seqlens", (B,))
    _same_device(q, (k_cache, "k_cache"), (v_cache, "v_cache"), (o, "o"), (lse, "lse"),
                 (seqlens, "seqlens"))
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    check(load().attn_decode_noalloc(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                                     o.data_ptr(), lse.data_ptr() if lse is not None else None,
                                     seqlens.data_ptr() if seqlens is not None else None,
                                     B, Hq, Hkv, Lmax, d, float(scale), int(window_left),
                                     int(num_splits), _stream_handle(stream)))
    return o, lse


def attn_device_status(stream=None) -> int:
    """Synchronise the stream, read and clear the device timeout word (0 = ok)."""
    return int(load().attn_device_status(_stream_handle(stream)))


def attn_last_error() -> str:
    msg = load().attn_last_error()
    return msg.decode() if msg else ""


def attn_launch_count() -> int:
    return int(load().attn_launch_count())
