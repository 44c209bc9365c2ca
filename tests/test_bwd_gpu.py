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
