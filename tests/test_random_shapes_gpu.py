"""GPU parity on seeded random shapes, against the fp64 oracle.

The fixed-shape tests pick the edge cases by hand; this file draws shapes at
random (seeded, so every run checks the same ones): batch, head counts and
group sizes (including odd groups and MQA), query and key lengths that are not
multiples of the tile (including Nq != Nk and a single key or query), head
dimension 64 or 128, causal or not, with or without a window, bf16 or fp32
output; decode with random lengths, windows and split counts; the backward on
small random shapes. Every output is compared element by element, with the
tolerances of the other parity tests.
"""

import random

import numpy as np
import pytest
import torch

import attn_inputs as ai
import oracle
from parity import assert_close, cuda

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from exact_softmax_attention_03_b200 import build
    build.build()


def _fwd_cases(n, seed):
    rng = random.Random(seed)
    cases = []
    for i in range(n):
        G = rng.choice([1, 1, 2, 3, 4, 8])
        Hkv = rng.randint(1, 3)
        B = rng.randint(1, 3)
        Nq = rng.choice([1, rng.randint(2, 130), rng.randint(100, 700), rng.randint(100, 700)])
        Nk = Nq if rng.random() < 0.6 else rng.choice([1, rng.randint(2, 700), rng.randint(2, 700)])
        d = rng.choice([64, 128])
        causal = rng.random() < 0.7
        wl = -1 if rng.random() < 0.5 else rng.randint(0, 400)
        f32 = rng.random() < 0.2
        cases.append((B, G * Hkv, Hkv, Nq, Nk, d, causal, wl, f32, 1000 + i))
    return cases


@pytest.mark.parametrize("case", _fwd_cases(24, seed=2026), ids=lambda c: "-".join(map(str, c[:9])))
def test_forward_random_shapes(case):
    import exact_softmax_attention_03_b200 as ea
    B, Hq, Hkv, Nq, Nk, d, causal, wl, f32, seed = case
    q, k, v = ai.make_qkv(B, Hq, Hkv, Nq, Nk, d, seed=seed)
    qg, kg, vg = cuda(q, k, v)
    lse = torch.full((B, Hq, Nq), 3.0, device="cuda")
    fn = ea.attn_fwd_f32o if f32 else ea.attn_fwd
    o, _ = fn(qg, kg, vg, lse=lse, causal=causal, window_left=wl)
    assert ea.attn_device_status() == 0
    O, L = oracle.oracle_attention(q, k, v, causal=causal, window_left=wl)
    assert_close(o, O, lse, L, what=case)


def _dec_cases(n, seed):
    rng = random.Random(seed)
    cases = []
    for i in range(n):
        G = rng.choice([1, 2, 4, 8])
        Hkv = rng.randint(1, 4)
        B = rng.randint(1, 9)
        L = rng.randint(1, 3000)
        d = rng.choice([64, 128])
        wl = -1 if rng.random() < 0.6 else rng.randint(0, 1000)
        splits = rng.choice([0, 0, 1, 2, 5])
        ragged = rng.random() < 0.5
        cases.append((B, G * Hkv, Hkv, L, d, wl, splits, ragged, 2000 + i))
    return cases


@pytest.mark.parametrize("case", _dec_cases(12, seed=2027), ids=lambda c: "-".join(map(str, c[:8])))
def test_decode_random_shapes(case):
    import exact_softmax_attention_03_b200 as ea
    B, Hq, Hkv, L, d, wl, splits, ragged, seed = case
    q, kc, vc = ai.make_decode(B, Hq, Hkv, L, d, seed=seed)
    sl = ai.ragged_seqlens(B, L, seed=seed) if ragged else None
    qg, kg, vg = cuda(q, kc, vc)
    lse = torch.full((B, Hq), 5.0, device="cuda")
    o, _ = ea.attn_decode(qg, kg, vg, lse=lse, seqlens=None if sl is None else sl.cuda(),
                          window_left=wl, num_splits=splits)
    assert ea.attn_device_status() == 0
    O, Lr = oracle.oracle_decode(q, kc, vc, sl, window_left=wl)
    assert_close(o, O, lse, Lr, what=case)


def _bwd_cases(n, seed):
    rng = random.Random(seed)
    cases = []
    for i in range(n):
        G = rng.choice([1, 2, 3])
        Hkv = rng.randint(1, 2)
        N = rng.randint(60, 420)
        Nk = N if rng.random() < 0.7 else rng.randint(60, 420)
        d = rng.choice([64, 128])
        causal = rng.random() < 0.7
        wl = -1 if rng.random() < 0.6 else rng.randint(0, 300)
        cases.append((1, G * Hkv, Hkv, N, Nk, d, causal, wl, 3000 + i))
    return cases


@pytest.mark.parametrize("case", _bwd_cases(6, seed=2028), ids=lambda c: "-".join(map(str, c[:8])))
def test_backward_random_shapes(case):
    import exact_softmax_attention_03_b200 as ea
    B, Hq, Hkv, Nq, Nk, d, causal, wl, seed = case
    q, k, v = ai.make_qkv(B, Hq, Hkv, Nq, Nk, d, seed=seed)
    do = ai.make_dout(B, Nq, Hq, d, seed=seed + 1)
    qg, kg, vg, dog = cuda(q, k, v, do)
    lse = torch.empty(B, Hq, Nq, device="cuda")
    o, _ = ea.attn_fwd(qg, kg, vg, lse=lse, causal=causal, window_left=wl)
    got = ea.attn_bwd(qg, kg, vg, o, lse, dog, causal=causal, window_left=wl)
    assert ea.attn_device_status() == 0
    ref = oracle.oracle_attention_backward(q, k, v, do, causal=causal, window_left=wl)
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        g = g.float().cpu().numpy().astype(np.float64)
        assert np.isfinite(g).all(), (case, name)
        rel = np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-30)
        mx = np.abs(g - r).max() / max(np.abs(r).max(), 1e-30)
        assert rel <= 5e-3 and mx <= 1.5e-2, (case, name, rel, mx)
