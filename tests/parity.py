"""Shared comparison helpers for the GPU parity tests.

Tolerances for bf16 inputs with fp32 accumulation against the fp64 oracle on
identical inputs: max |ΔO| <= 2e-2, relative L2 of O <= 5e-3, max |ΔLSE| <= 1e-3.
Rows with no allowed key must match exactly: O = 0 and LSE = -inf.
"""

import numpy as np
import torch

MAX_ABS = 2e-2
REL_L2 = 5e-3
LSE_ABS = 1e-3


def errors(o_gpu, o_ref, lse_gpu=None, lse_ref=None):
    o = o_gpu.detach().float().cpu().numpy().astype(np.float64)
    r = np.asarray(o_ref, dtype=np.float64)
    assert o.shape == r.shape, (o.shape, r.shape)
    assert np.isfinite(o).all(), "non-finite output"
    diff = o - r
    out = {
        "max_abs": float(np.abs(diff).max()) if diff.size else 0.0,
        "rel_l2": float(np.linalg.norm(diff) / max(np.linalg.norm(r), 1e-30)),
    }
    if lse_gpu is not None:
        lg = lse_gpu.detach().float().cpu().numpy().astype(np.float64)
        lr = np.asarray(lse_ref, dtype=np.float64)
        assert lg.shape == lr.shape
        ninf_g, ninf_r = np.isneginf(lg), np.isneginf(lr)
        assert (ninf_g == ninf_r).all(), "-inf pattern of LSE differs"
        fin = ~ninf_r
        assert np.isfinite(lg[fin]).all()
        out["lse_abs"] = float(np.abs(lg[fin] - lr[fin]).max()) if fin.any() else 0.0
    return out


def assert_close(o_gpu, o_ref, lse_gpu=None, lse_ref=None, what=""):
    e = errors(o_gpu, o_ref, lse_gpu, lse_ref)
    assert e["max_abs"] <= MAX_ABS, (what, e)
    assert e["rel_l2"] <= REL_L2, (what, e)
    if "lse_abs" in e:
        assert e["lse_abs"] <= LSE_ABS, (what, e)
    return e


def cuda(*ts):
    return [t.cuda() for t in ts]


def sample_rows(n, k, seed):
    """k distinct row indices of [0, n) that always include 0 and n - 1."""
    g = torch.Generator().manual_seed(seed)
    pick = torch.randperm(n, generator=g)[:max(0, k - 2)].tolist()
    return sorted(set(pick) | {0, n - 1})


def backward_of_group(q, k, v, dout, b, hk, causal, window_left):
    """Oracle dQ, dK, dV of one (batch, K/V head) and its group of query heads.

    The gradients of a K/V head and the dQ of its query heads depend only on
    that group's inputs, so a full-size problem can be checked one group at a
    time. Returns (dQ [Nq, G, d], dK [Nk, d], dV [Nk, d]) in fp64.
    """
    import oracle
    G = q.shape[2] // k.shape[2]
    hs = slice(hk * G, (hk + 1) * G)
    dq, dk, dv = oracle.oracle_attention_backward(
        q[b:b + 1, :, hs], k[b:b + 1, :, hk:hk + 1], v[b:b + 1, :, hk:hk + 1],
        dout[b:b + 1, :, hs], causal=causal, window_left=window_left)
    return dq[0], dk[0, :, 0], dv[0, :, 0]
