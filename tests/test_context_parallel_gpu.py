"""GPU parity of sequence-sharded attention and of the merge kernel.

The ranks of a world of R are emulated in one process (each call is what a
rank computes after the all-gather); the concatenated chunks must equal the
fp64 oracle on the whole sequence. The merge kernel is checked against the
oracle's merge rule on random parts, including rows no part saw a key for.
"""

import numpy as np
import pytest
import torch

import attn_inputs as ai
import oracle
from parity import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from exact_softmax_attention_03_b200 import build
    build.build()


@pytest.mark.parametrize("R,C,Hq,Hkv,d,causal", [(2, 256, 4, 4, 128, True),
                                                 (3, 200, 8, 2, 128, True),
                                                 (4, 130, 4, 1, 64, True),
                                                 (3, 160, 4, 2, 128, False)])
def test_sharded_sequence_equals_whole(R, C, Hq, Hkv, d, causal):
    import exact_softmax_attention_03_b200 as ea
    from exact_softmax_attention_03_b200.context_parallel import context_parallel_local
    q, k, v = ai.make_qkv(2, Hq, Hkv, R * C, R * C, d)
    qc = [q[:, r * C:(r + 1) * C].contiguous().cuda() for r in range(R)]
    kc = [k[:, r * C:(r + 1) * C].contiguous().cuda() for r in range(R)]
    vc = [v[:, r * C:(r + 1) * C].contiguous().cuda() for r in range(R)]
    outs, lses = [], []
    for r in range(R):
        o, lse = context_parallel_local(qc[r], kc, vc, r, causal=causal)
        outs.append(o)
        lses.append(lse)
    assert ea.attn_device_status() == 0
    O, L = oracle.oracle_attention(q, k, v, causal=causal)
    assert_close(torch.cat(outs, dim=1), O, torch.cat(lses, dim=2), L, what=(R, C, causal))


@pytest.mark.parametrize("R,d,Nq", [(3, 128, 17), (5, 64, 17), (20, 128, 17), (1, 128, 70),
                                    (2, 64, 70), (4, 128, 70), (8, 128, 33), (9, 64, 64),
                                    (64, 128, 40)])
def test_merge_kernel_against_merge_rule(R, d, Nq):
    import exact_softmax_attention_03_b200 as ea
    g = torch.Generator().manual_seed(7)
    B, H = 2, 4
    op = torch.randn(R, B, Nq, H, d, generator=g)
    lp = torch.randn(R, B, H, Nq, generator=g) * 3
    lp[min(1, R - 1), 0, 2, 5] = -float("inf")     # one part saw no key for this row
    lp[:, 1, 3, 7] = -float("inf")                 # no part saw a key
    o, lse = ea.attn_merge(op.cuda(), lp.cuda(), lse=torch.empty(B, H, Nq, device="cuda"))
    assert ea.attn_device_status() == 0
    O = np.zeros((B, Nq, H, d))
    Lr = np.zeros((B, H, Nq))
    for b in range(B):
        for qq in range(Nq):
            for h in range(H):
                parts = [(float(lp[r, b, h, qq]), 1.0, op[r, b, qq, h].double().numpy())
                         for r in range(R)]
                O[b, qq, h], Lr[b, h, qq] = oracle.merge_partials(parts)
    assert_close(o, O, lse, Lr, what="merge")
    assert (o[1, 7, 3].float() == 0).all() and torch.isneginf(lse[1, 3, 7])
