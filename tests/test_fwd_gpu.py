"""GPU parity of attn_fwd / attn_fwd_f32o against the fp64 oracle.

Small problems are compared element by element over every output; the full
workload sizes (MHA 2K and 8K causal, GQA sliding window at 32K) run in the
same launch configuration the bench times and are compared on sampled rows
that the oracle computes one by one.
"""

import numpy as np
import pytest
import torch

import attn_inputs as ai
import oracle
from parity import assert_close, cuda, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from exact_softmax_attention_03_b200 import build
    build.build()


def run_fwd(q, k, v, causal, wl, f32=False, scale=None, with_lse=True):
    import exact_softmax_attention_03_b200 as ea
    qg, kg, vg = cuda(q, k, v)
    B, Nq, Hq, d = q.shape
    lse = torch.full((B, Hq, Nq), 7.0, device="cuda") if with_lse else None
    fn = ea.attn_fwd_f32o if f32 else ea.attn_fwd
    o, _ = fn(qg, kg, vg, lse=lse, causal=causal, window_left=wl, scale=scale)
    assert ea.attn_device_status() == 0
    return o, lse


def check_full(shape, causal, wl, f32=False, seed=ai.SEED_Q, scale=None):
    B, Hq, Hkv, Nq, Nk, d = shape
    q, k, v = ai.make_qkv(B, Hq, Hkv, Nq, Nk, d, seed)
    o, lse = run_fwd(q, k, v, causal, wl, f32=f32, scale=scale)
    O, L = oracle.oracle_attention(q, k, v, causal=causal, window_left=wl, scale=scale)
    return assert_close(o, O, lse, L, what=(shape, causal, wl))


@pytest.mark.parametrize("causal", [False, True])
def test_tiny_workload_fp32_out(causal):
    w = ai.TINY_CAUSAL if causal else ai.TINY
    check_full((w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d), w.causal, w.window_left, f32=True)


SHAPES = [
    # (B, Hq, Hkv, Nq, Nk, d), causal, window_left
    ((1, 2, 2, 1, 1, 128), True, -1),
    ((1, 2, 2, 127, 127, 128), True, -1),
    ((1, 2, 2, 129, 129, 128), False, -1),
    ((2, 4, 4, 1000, 1000, 128), True, -1),
    ((1, 2, 2, 100, 300, 128), True, -1),        # Nq < Nk: bottom-right alignment
    ((1, 2, 2, 300, 100, 128), True, -1),        # Nq > Nk: leading rows see no key
    ((1, 4, 1, 515, 515, 128), True, 0),         # MQA, window of one key
    ((1, 4, 1, 515, 515, 128), True, 1),
    ((1, 4, 1, 515, 515, 128), True, 127),
    ((1, 4, 1, 515, 515, 128), True, 128),
    ((1, 4, 1, 515, 515, 128), True, 129),
    ((1, 8, 2, 384, 384, 128), True, 200),       # GQA, head pairs share K/V tiles
    ((1, 6, 2, 300, 300, 64), True, -1),         # odd group size (3)
    ((1, 4, 4, 257, 257, 64), False, 50),        # window without causal
    ((2, 2, 1, 640, 640, 64), True, -1),
    ((1, 1, 1, 2048, 2048, 128), False, -1),
    ((1, 2, 2, 700, 1500, 128), False, 300),
    ((1, 2, 2, 1, 4000, 128), True, -1),         # one query at the end of a long key set
    ((1, 16, 2, 257, 257, 128), True, 100),      # GQA group of 8: four head pairs per K/V head
    ((2, 32, 1, 200, 200, 64), False, -1),       # MQA, 32 query heads on one K/V head
    ((3, 4, 2, 129, 385, 64), True, 64),         # ragged, Nq < Nk, window, d = 64
]


@pytest.mark.parametrize("shape,causal,wl", SHAPES)
def test_parity_shapes(shape, causal, wl):
    check_full(shape, causal, wl)


def test_parity_fp32_out_ragged():
    check_full((1, 4, 2, 333, 333, 128), True, 100, f32=True)


def test_custom_scale():
    check_full((1, 2, 2, 200, 200, 128), True, -1, scale=0.3)


def test_no_lse_pointer():
    q, k, v = ai.make_qkv(1, 2, 2, 256, 256, 128)
    o, _ = run_fwd(q, k, v, True, -1, with_lse=False)
    O, _ = oracle.oracle_attention(q, k, v, causal=True)
    assert_close(o, O)


def test_fully_masked_rows_are_exact_zero_and_minus_inf():
    q, k, v = ai.make_qkv(1, 2, 2, 300, 100, 128)
    o, lse = run_fwd(q, k, v, True, -1)
    assert (o[:, :200].float() == 0).all()
    assert torch.isneginf(lse[:, :, :200]).all()
    assert torch.isfinite(lse[:, :, 200:]).all()


def test_deterministic_bitwise():
    q, k, v = ai.make_qkv(2, 8, 2, 700, 700, 128)
    o1, l1 = run_fwd(q, k, v, True, 300)
    o2, l2 = run_fwd(q, k, v, True, 300)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_constant_v_gives_constant_output():
    q, k, _ = ai.make_qkv(1, 4, 4, 500, 500, 128)
    v = torch.full_like(k, 0.625)
    o, _ = run_fwd(q, k, v, True, -1)
    assert torch.allclose(o.float(), torch.full_like(o.float(), 0.625), atol=4e-3)


FULL = [ai.MHA_2K, ai.MHA_8K, ai.GQA_SWA_32K]


def _head(t, b, h):
    return t[b:b + 1, :, h:h + 1]


@pytest.mark.parametrize("w", FULL, ids=lambda w: w.name)
def test_full_size_whole_head_and_late_rows(w):
    """One launch at the full workload size, in the bench's configuration.

    * One whole (batch, head) is compared element by element with the oracle
      (every row block of that head, so every position in the work order);
      at N = 32768, where one head costs the fp64 oracle about a minute, two
      spans of 512 rows of it (the middle and the end).
    * The shortest causal row blocks run last in the kernel's work order
      (longest rows first); rows of the first 256 and of the last 256 query
      positions are sampled on 12 more heads, plus 24 rows anywhere.
    """
    q, k, v = ai.make_for(w)
    o, lse = run_fwd(q, k, v, w.causal, w.window_left)
    assert torch.isfinite(o.float()).all()
    assert torch.isfinite(lse).all()
    G = w.Hq // w.Hkv
    b, hq = w.B - 1, w.Hq - 1
    if w.Nq * w.Nk <= 8192 * 8192:
        O, L = oracle.oracle_attention(_head(q, b, hq), _head(k, b, hq // G),
                                       _head(v, b, hq // G), causal=w.causal,
                                       window_left=w.window_left)
        assert_close(o[b:b + 1, :, hq:hq + 1], O, lse[b:b + 1, hq:hq + 1], L,
                     what=(w.name, "whole head", b, hq))
    else:
        rows = list(range(w.Nq // 2, w.Nq // 2 + 512)) + list(range(w.Nq - 512, w.Nq))
        O, L = oracle.oracle_attention_rows(_head(q, b, hq), _head(k, b, hq // G),
                                            _head(v, b, hq // G), 0, 0, rows, causal=w.causal,
                                            window_left=w.window_left)
        assert_close(o[b, rows, hq], O, lse[b, hq, rows], L, what=(w.name, "row spans", b, hq))
    g = torch.Generator().manual_seed(99)
    for i in range(12):
        b = int(torch.randint(w.B, (1,), generator=g))
        hq = int(torch.randint(w.Hq, (1,), generator=g))
        early = torch.randint(0, 256, (8,), generator=g).tolist()
        late = torch.randint(w.Nq - 256, w.Nq, (4,), generator=g).tolist()
        rows = sorted(set(early + late + sample_rows(w.Nq, 24, seed=1000 * b + hq)))
        O, L = oracle.oracle_attention_rows(_head(q, b, hq), _head(k, b, hq // G),
                                            _head(v, b, hq // G), 0, 0, rows, causal=w.causal,
                                            window_left=w.window_left)
        assert_close(o[b, rows, hq], O, lse[b, hq, rows], L, what=(w.name, b, hq))


def test_head_grouped_gqa_causal_sampled_rows():
    """GQA causal without a window at N = 32768 (Hq32 Hkv8): its K/V (128 MB) is
    above L2, so the work list runs in head groups (4 of 4 head pairs each) with
    the rotated per-group assignment. Sampled rows of 6 heads, including the
    shortest causal rows (they run last within each group)."""
    B, Hq, Hkv, N, d = 1, 32, 8, 32768, 128
    q, k, v = ai.make_qkv(B, Hq, Hkv, N, N, d, seed=ai.SEED_Q + 90)
    o, lse = run_fwd(q, k, v, True, -1)
    G = Hq // Hkv
    g = torch.Generator().manual_seed(5)
    for hq in (0, 5, 10, 17, 26, 31):
        early = torch.randint(0, 256, (6,), generator=g).tolist()
        rows = sorted(set(early + sample_rows(N, 12, seed=hq)))
        O, L = oracle.oracle_attention_rows(_head(q, 0, hq), _head(k, 0, hq // G),
                                            _head(v, 0, hq // G), 0, 0, rows, causal=True)
        assert_close(o[0, rows, hq], O, lse[0, hq, rows], L, what=("grouped GQA", hq))


def _scaled_keys(k, factor_of_key):
    k = k.float().clone()
    for j in range(k.shape[1]):
        f = factor_of_key(j)
        if f != 1.0:
            k[:, j] *= f
    return k.to(torch.bfloat16)


def test_scores_growing_across_blocks_force_a_fresh_max():
    # Key blocks are visited from the last one backwards; the early keys get
    # scores tens of log2 units above everything seen before, so the running
    # max (reused without a max pass) must be refreshed exactly.
    q, k, v = ai.make_qkv(1, 2, 2, 640, 640, 128)
    k = _scaled_keys(k, lambda j: 90.0 if j < 128 else (30.0 if j < 256 else 1.0))
    for causal in (True, False):
        o, lse = run_fwd(q, k, v, causal, -1)
        O, L = oracle.oracle_attention(q, k, v, causal=causal)
        assert_close(o, O, lse, L, what=("growing", causal))


def test_overflow_in_second_half_of_a_block():
    # Only keys 64..127 of block 1 are huge: the first half of that block goes
    # out with the old max and the second half has to rescale after it.
    q, k, v = ai.make_qkv(2, 4, 2, 512, 512, 128)
    k = _scaled_keys(k, lambda j: 60.0 if 192 <= j < 256 else 1.0)
    for causal, wl in ((True, -1), (False, -1), (True, 300)):
        o, lse = run_fwd(q, k, v, causal, wl)
        O, L = oracle.oracle_attention(q, k, v, causal=causal, window_left=wl)
        assert_close(o, O, lse, L, what=("second half", causal, wl))


def test_tensors_past_4_gib():
    """Q, K, V and O of 4.56 GB each (B1 N131072 H136 d128: more than 2^31
    elements, byte offsets past 2^32 in every tensor), causal with a window of
    128 keys so the launch stays short. Rows at the start, in the middle and at
    the end (past 2^32 bytes) of three heads are compared element by element
    with the oracle; every output must be finite."""
    import exact_softmax_attention_03_b200 as ea
    B, H, N, d, wl = 1, 136, 131072, 128, 127
    q, k, v = ai.make_qkv_on("cuda", B, H, H, N, N, d, seed=ai.SEED_Q + 60)
    assert q.numel() > 2 ** 31 and q.numel() * q.element_size() > 2 ** 32
    lse = torch.empty(B, H, N, device="cuda")
    o, _ = ea.attn_fwd(q, k, v, lse=lse, causal=True, window_left=wl)
    assert ea.attn_device_status() == 0
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()
    rows = list(range(0, 64)) + list(range(N // 2 - 32, N // 2 + 32)) + list(range(N - 64, N))
    for h in (0, 67, H - 1):
        O, L = oracle.oracle_attention_rows(_head(q, 0, h).cpu(), _head(k, 0, h).cpu(),
                                            _head(v, 0, h).cpu(), 0, 0, rows, causal=True,
                                            window_left=wl)
        assert_close(o[0, rows, h], O, lse[0, h, rows], L, what=("past 4 GiB", h))
    del q, k, v, o
    torch.cuda.empty_cache()
