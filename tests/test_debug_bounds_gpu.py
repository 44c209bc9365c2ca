"""The bounds-checking debug build (libattn_debug.so) on the small parity cases.

That build checks, in every kernel, each computed global-memory index against
the extent of the buffer it addresses, and at the end of each CTA that the
pipeline roles counted the same stages; a failed check skips the access and
is reported by attn_device_status() as ATTN_ERR_INTERNAL. It stands in for a
memory checker, which cannot run on these machines.

Here the small forward (plain, windowed, GQA, packed), decode (contiguous and
paged), backward, merge and random-shape parity tests run in a child process against the
debug build (ATTN_LIBRARY=debug): every call must pass parity with the fp64
oracle and leave the status word clear. So does the full-size MHA causal
N = 8192 forward, the one workload here whose work list runs in head groups.
Only valid inputs are used: a check that fails on a valid input is a bug in
the kernel or in the check.
"""

import os
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.gpu

CASES = [
    "tests/test_fwd_gpu.py::test_parity_shapes",
    "tests/test_fwd_gpu.py::test_tiny_workload_fp32_out",
    "tests/test_fwd_gpu.py::test_fully_masked_rows_are_exact_zero_and_minus_inf",
    "tests/test_fwd_varlen_gpu.py",
    "tests/test_decode_gpu.py",
    "tests/test_decode_paged_gpu.py",
    "tests/test_bwd_gpu.py",
    "tests/test_context_parallel_gpu.py",
    "tests/test_random_shapes_gpu.py",
]


@pytest.fixture(scope="module")
def debug_lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from exact_softmax_attention_03_b200 import build
    return build.build(debug=True)


def test_debug_build_reports_itself(debug_lib):
    code = ("import exact_softmax_attention_03_b200._lib as L; lib = L.load(); "
            "print(L.LIB_PATH, lib.attn_debug_checks())")
    env = dict(os.environ, ATTN_LIBRARY="debug")
    res = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True,
                         text=True, timeout=120)
    assert res.returncode == 0, res.stderr[-2000:]
    path, flag = res.stdout.split()
    assert path.endswith("libattn_debug.so") and flag == "1"


def test_small_parity_cases_pass_under_the_debug_build(debug_lib):
    env = dict(os.environ, ATTN_LIBRARY="debug")
    cmd = [sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-k", "not full_size",
           "-p", "no:cacheprovider", *CASES]
    res = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=1800)
    assert res.returncode == 0, (res.stdout[-4000:], res.stderr[-2000:])
    assert " passed" in res.stdout


def test_full_size_head_grouped_forward_under_the_debug_build(debug_lib):
    env = dict(os.environ, ATTN_LIBRARY="debug")
    cmd = [sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-k", "N8192",
           "-p", "no:cacheprovider", "tests/test_fwd_gpu.py::test_full_size_whole_head_and_late_rows"]
    res = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=1800)
    assert res.returncode == 0, (res.stdout[-4000:], res.stderr[-2000:])
    assert "1 passed" in res.stdout
