"""Failure detection without faulting the GPU.

Every wait in the kernels is bounded. attn_selftest_wait_timeout launches a
kernel whose wait can never complete; the kernel must give up after about a
second, report ATTN_ERR_TIMEOUT through the status word, and leave the context
usable: a normal forward call afterwards is correct and reports no timeout.
"""

import time

import pytest
import torch

import attn_inputs as ai
import oracle
from parity import assert_close, cuda

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from exact_softmax_attention_03_b200 import _lib, build
    build.build()
    return _lib.load()


def test_bounded_wait_times_out_and_reports(lib):
    from exact_softmax_attention_03_b200 import _lib
    stream = torch.cuda.current_stream().cuda_stream
    assert lib.attn_device_status(stream) == _lib.ATTN_OK          # clean start
    t0 = time.perf_counter()
    assert lib.attn_selftest_wait_timeout(stream) == _lib.ATTN_OK
    assert lib.attn_device_status(stream) == _lib.ATTN_ERR_TIMEOUT
    elapsed = time.perf_counter() - t0
    assert 0.5 < elapsed < 10.0                                    # ~1 s limit
    assert lib.attn_device_status(stream) == _lib.ATTN_OK          # cleared by the read


def test_context_stays_usable_after_a_timeout(lib):
    import exact_softmax_attention_03_b200 as ea
    from exact_softmax_attention_03_b200 import _lib
    stream = torch.cuda.current_stream().cuda_stream
    assert lib.attn_selftest_wait_timeout(stream) == _lib.ATTN_OK
    assert lib.attn_device_status(stream) == _lib.ATTN_ERR_TIMEOUT
    q, k, v = ai.make_qkv(1, 2, 2, 300, 300, 128)
    qg, kg, vg = cuda(q, k, v)
    lse = torch.empty(1, 2, 300, device="cuda")
    o, _ = ea.attn_fwd(qg, kg, vg, lse=lse, causal=True)
    assert ea.attn_device_status() == 0
    O, L = oracle.oracle_attention(q, k, v, causal=True)
    assert_close(o, O, lse, L)
