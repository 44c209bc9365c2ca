"""GPU parity of attn_bwd (dQ, dK, dV) against the fp64 backward oracle.

The forward output and LSE come from attn_fwd on the same inputs, as in
training. Tolerances: the kernel rounds P and dS to bf16 before the products
(relative error 2^-9 each, as P in the forward) and accumulates in fp32, so
the forward's relative-L2 bound of 5e-3 applies to dQ, dK and dV; every
element must lie within 1.5e-2 of the largest reference magnitude (measured:
about 2.5e-3 and 4.6e-3).
"""

import numpy as np
import pytest
import torch

import attn_inputs as ai
import oracle
from parity import backward_of_group, cuda

pytestmark = pytest.mark.gpu

REL_L2 = {"dq": 5e-3, "dk": 5e-3, "dv": 5e-3}
MAX_REL = 1.5e-2


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from exact_softmax_attention_03_b200 import build
    build.build()


def gpu_bwd(B, Hq, Hkv, Nq, Nk, d, causal, wl):
    """Inputs (CPU, bf16) and the GPU gradients, with O and LSE from attn_fwd."""
    import exact_softmax_attention_03_b200 as ea
    q, k, v = ai.make_qkv(B, Hq, Hkv, Nq, Nk, d)
    do = ai.make_dout(B, Nq, Hq, d)
    qg, kg, vg, dog = cuda(q, k, v, do)
    lse = torch.empty(B, Hq, Nq, device="cuda")
    o, _ = ea.attn_fwd(qg, kg, vg, lse=lse, causal=causal, window_left=wl)
    dq, dk, dv = ea.attn_bwd(qg, kg, vg, o, lse, dog, causal=causal, window_left=wl)
    assert ea.attn_device_status() == 0
    return (q, k, v, do), (dq, dk, dv)


def run_bwd(B, Hq, Hkv, Nq, Nk, d, causal, wl):
    (q, k, v, do), got = gpu_bwd(B, Hq, Hkv, Nq, Nk, d, causal, wl)
    ref = oracle.oracle_attention_backward(q, k, v, do, causal=causal, window_left=wl)
    return got, ref


def compare(got, ref, what):
    """rel-L2 and largest error relative to the largest reference magnitude."""
    errs = {}
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        g = g.float().cpu().numpy().astype(np.float64)
        assert np.isfinite(g).all(), name
        scale = max(np.abs(r).max(), 1e-30)
        e = {"rel_l2": float(np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-30)),
             "max_rel": float(np.abs(g - r).max() / scale)}
        errs[name] = e
        print(what, name, e)
    for name, e in errs.items():
        assert e["rel_l2"] <= REL_L2[name], (what, name, errs)
        assert e["max_rel"] <= MAX_REL, (what, name, errs)
    return errs


def check(shape, causal, wl):
    got, ref = run_bwd(*shape, causal, wl)
    return compare(got, ref, (shape, causal, wl))


SHAPES = [
    # (B, Hq, Hkv, Nq, Nk, d), causal, window_left
    ((1, 2, 2, 128, 128, 128), True, -1),
    ((1, 2, 2, 256, 256, 128), False, -1),
    ((2, 4, 2, 300, 300, 128), True, -1),      # GQA, ragged tail
    ((1, 2, 2, 200, 500, 128), True, -1),      # Nq < Nk (bottom-right)
    ((1, 4, 1, 384, 384, 128), True, 100),     # MQA, window
    ((1, 2, 2, 257, 257, 64), True, -1),       # d = 64
    ((1, 2, 2, 1024, 1024, 128), True, -1),    # many blocks per key block
    ((1, 2, 2, 160, 333, 64), False, 40),      # window without causal, d = 64
    # mask edges inside one query half of a block only (each half of a block's
    # queries is formed by its own elementwise warps)
    ((1, 2, 2, 192, 192, 128), True, 100),
    ((2, 4, 2, 320, 200, 64), True, 70),       # rows without keys, GQA, d = 64
    ((1, 2, 2, 130, 450, 128), False, 90),     # window without causal, Nq < Nk
]


@pytest.mark.parametrize("shape,causal,wl", SHAPES)
def test_backward_parity(shape, causal, wl):
    check(shape, causal, wl)


def test_rows_without_keys_get_zero_query_gradient():
    got, _ = run_bwd(1, 2, 2, 300, 100, 128, True, -1)
    dq = got[0]
    assert (dq[:, :200].float() == 0).all()


FULL = [
    # the backward workload the bench times (MHA causal B4 H32 N2048 d128), and a
    # GQA windowed problem of the same size; same launch configuration
    ((4, 32, 32, 2048, 2048, 128), True, -1),
    ((2, 32, 8, 2048, 2048, 128), True, 512),
]


@pytest.mark.parametrize("shape,causal,wl", FULL)
def test_full_size_sampled_groups(shape, causal, wl):
    B, Hq, Hkv, Nq, Nk, d = shape
    G = Hq // Hkv
    (q, k, v, do), (dq, dk, dv) = gpu_bwd(*shape, causal, wl)
    for t in (dq, dk, dv):
        assert torch.isfinite(t.float()).all()
    g = torch.Generator().manual_seed(7)
    picks = [(0, 0), (B - 1, Hkv - 1),
             (int(torch.randint(B, (1,), generator=g)), int(torch.randint(Hkv, (1,), generator=g)))]
    for b, hk in picks:
        ref = backward_of_group(q, k, v, do, b, hk, causal, wl)
        got = (dq[b, :, hk * G:(hk + 1) * G], dk[b, :, hk], dv[b, :, hk])
        compare(got, ref, (shape, causal, wl, b, hk))


def test_tensors_past_4_gib():
    """Q, K, V, O, dO and the three gradients of 4.56 GB each (B1 N131072 H136
    d128: more than 2^31 elements, byte offsets past 2^32), causal with a
    window of 128 keys. With that window a span of rows and keys is a closed
    problem away from its edges: the oracle's backward of the span gives the
    exact dQ of its rows that see 128 keys inside it and the exact dK, dV of
    its keys whose 128 queries lie inside it. Spans at the start, in the middle
    and at the end (past 2^32 bytes) of two heads are compared."""
    import exact_softmax_attention_03_b200 as ea
    B, H, N, d, wl, S = 1, 136, 131072, 128, 127, 1024
    q, k, v = ai.make_qkv_on("cuda", B, H, H, N, N, d, seed=ai.SEED_Q + 62)
    do = ai.make_dout_on("cuda", B, N, H, d, seed=ai.SEED_Q + 63)
    assert q.numel() > 2 ** 31 and q.numel() * q.element_size() > 2 ** 32
    lse = torch.empty(B, H, N, device="cuda")
    o, _ = ea.attn_fwd(q, k, v, lse=lse, causal=True, window_left=wl)
    dq, dk, dv = ea.attn_bwd(q, k, v, o, lse, do, causal=True, window_left=wl)
    assert ea.attn_device_status() == 0
    for t in (dq, dk, dv):
        assert torch.isfinite(t).all()
    del o
    for h in (0, H - 1):
        for s0 in (0, N // 2 - S // 2, N - S):
            s1 = s0 + S
            sl = (slice(0, 1), slice(s0, s1), slice(h, h + 1))
            rq, rk, rv = oracle.oracle_attention_backward(q[sl].cpu(), k[sl].cpu(), v[sl].cpu(),
                                                          do[sl].cpu(), causal=True, window_left=wl)
            r_lo = s0 if s0 == 0 else s0 + wl                 # rows whose keys lie in the span
            k_lo = s0 if s0 == 0 else s0 + wl                 # keys whose queries' sums are exact
            k_hi = s1 if s1 == N else s1 - wl                 # keys whose queries lie in the span
            got = (dq[0, r_lo:s1, h], dk[0, k_lo:k_hi, h], dv[0, k_lo:k_hi, h])
            ref = (rq[0, r_lo - s0:, 0], rk[0, k_lo - s0:k_hi - s0, 0], rv[0, k_lo - s0:k_hi - s0, 0])
            compare(got, ref, ("past 4 GiB", h, s0))
    del q, k, v, do, dq, dk, dv
    torch.cuda.empty_cache()
