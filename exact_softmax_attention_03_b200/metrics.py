"""Work and traffic counts used to turn measured times into throughput.

* Mask-adjusted FLOPs: ``4 * d * sum over (b, hq) of allowed (i, j) pairs``
  (one multiply-add per element for Q·Kᵀ and one for P·V). "Attention Is
  O(n²): FlashAttention vs Linear Attention", section "Why Attention Is
  O(n²)", counts ``2 * n² * d`` per head for the score product alone; the P·V
  product doubles it.
* Algorithmic HBM bytes of the tiled forward pass: read Q, K, V once and write
  O once (same page, section "What FLOPs Can't Be Avoided"), plus the fp32
  log-sum-exp row statistics (section "FlashAttention — Same FLOPs, Linear
  Memory").
* KV-cache bytes: ``2 (K and V) x layers x kv_heads x head_dim x seq_len x
  bytes`` ("Modern Attention: MQA, GQA, FlashAttention, Sliding Window and
  RoPE", section 1 "Why vanilla attention is expensive at inference").
"""

from __future__ import annotations

import numpy as np


def allowed_pairs_per_row(Nq: int, Nk: int, causal: bool, window_left: int) -> np.ndarray:
    """Number of keys each query row attends to (bottom-right causal alignment)."""
    i = np.arange(Nq, dtype=np.int64)
    qpos = i + (Nk - Nq)
    hi = np.minimum(qpos, Nk - 1) if causal else np.full(Nq, Nk - 1, dtype=np.int64)
    lo = np.maximum(qpos - window_left, 0) if window_left >= 0 else np.zeros(Nq, dtype=np.int64)
    return np.maximum(hi - lo + 1, 0)


def allowed_pairs(Nq: int, Nk: int, causal: bool, window_left: int) -> int:
    return int(allowed_pairs_per_row(Nq, Nk, causal, window_left).sum())


def attn_flops(B, Hq, Nq, Nk, d, causal, window_left) -> float:
    """Mask-adjusted algorithmic FLOPs of one forward call."""
    return 4.0 * d * B * Hq * allowed_pairs(Nq, Nk, causal, window_left)


def executed_tiles(Nq: int, Nk: int, causal: bool, window_left: int, bm: int = 128,
                   bn: int = 128) -> int:
    """128 x 128 score tiles a tile-skipping kernel computes for one head."""
    rows = allowed_pairs_per_row(Nq, Nk, causal, window_left)
    total = 0
    for r0 in range(0, Nq, bm):
        r1 = min(r0 + bm, Nq)
        qpos0, qpos1 = r0 + Nk - Nq, r1 - 1 + Nk - Nq
        hi = min(qpos1, Nk - 1) if causal else Nk - 1
        lo = max(qpos0 - window_left, 0) if window_left >= 0 else 0
        if rows[r0:r1].max() == 0 or hi < lo:
            continue
        total += hi // bn - lo // bn + 1
    return total


def attn_fwd_bytes(B, Hq, Hkv, Nq, Nk, d, out_bytes: int = 2, with_lse: bool = True) -> int:
    """Minimum HBM traffic of one forward call: Q, K, V read once; O (+LSE) written once."""
    qkv = 2 * (B * Nq * Hq * d + 2 * B * Nk * Hkv * d)
    o = out_bytes * B * Nq * Hq * d
    lse = 4 * B * Hq * Nq if with_lse else 0
    return qkv + o + lse


def decode_kv_bytes(seqlens, Hkv: int, d: int, window_left: int = -1, elem_bytes: int = 2) -> int:
    """K and V cache bytes a decode step must read (each visible key once)."""
    s = np.asarray(seqlens, dtype=np.int64).reshape(-1)
    if window_left >= 0:
        s = np.minimum(s, window_left + 1)
    return int(2 * s.sum() * Hkv * d * elem_bytes)


def decode_bytes(B, Hq, Hkv, seqlens, d, window_left=-1, with_lse=True) -> int:
    """KV read + q read + O write (+ LSE write) for one decode call."""
    kv = decode_kv_bytes(seqlens, Hkv, d, window_left)
    return kv + 2 * B * Hq * d * 2 + (4 * B * Hq if with_lse else 0)


def decode_flops(B, Hq, seqlens, d, window_left=-1) -> float:
    s = np.asarray(seqlens, dtype=np.int64).reshape(-1)
    if window_left >= 0:
        s = np.minimum(s, window_left + 1)
    return 4.0 * d * Hq * float(s.sum())


def kv_cache_bytes(layers: int, kv_heads: int, head_dim: int, seq_len: int,
                   elem_bytes: int = 2, batch: int = 1) -> int:
    """Dense KV-cache size of one model: 2 x layers x kv_heads x head_dim x seq_len x bytes."""
    return 2 * batch * layers * kv_heads * head_dim * seq_len * elem_bytes


def score_flops_one_product(seq_len: int, d_model: int, n_heads: int, n_layers: int) -> float:
    """The pages' table convention: 2 * n² * d_k per head (score product only)."""
    d_k = d_model // n_heads
    return 2.0 * seq_len * seq_len * d_k * n_heads * n_layers
