"""The Python binding's operand checks, on CPU.

Every entry point must refuse an output, LSE, length or table tensor of the
wrong shape, and operands on different devices, before anything reaches the
library: a smaller ``o`` or a ``seqlens`` shorter than the batch would
otherwise let a kernel write or read past the buffer. The tensors here are CPU
tensors that report a CUDA device, so the checks run without a GPU; none of
the calls may reach the library (its launch counter stays put).
"""

import pytest
import torch

import exact_softmax_attention_03_b200 as ea


class FakeCuda(torch.Tensor):
    """A CPU tensor that reports itself as living on ``cuda:<index>``."""

    index = 0

    @property
    def is_cuda(self):
        return True

    @property
    def device(self):
        return torch.device("cuda", type(self).index)


class FakeCuda1(FakeCuda):
    index = 1


def fake(shape, dtype=torch.bfloat16, other_device=False):
    cls = FakeCuda1 if other_device else FakeCuda
    return torch.zeros(shape, dtype=dtype).as_subclass(cls)


def refused(fn, *args, **kw):
    n0 = ea.attn_launch_count()
    with pytest.raises(ValueError, match=r"must have shape|is on cuda|must be \[|shaped like"):
        fn(*args, **kw)
    assert ea.attn_launch_count() == n0


B, Hq, Hkv, N, d = 2, 4, 2, 16, 64


def qkv():
    return (fake((B, N, Hq, d)), fake((B, N, Hkv, d)), fake((B, N, Hkv, d)))


def test_forward_checks_shapes_and_devices():
    q, k, v = qkv()
    refused(ea.attn_fwd, q, k, v, o=fake((B, N, Hq, d - 8)))
    refused(ea.attn_fwd, q, k, v, o=fake((B, N, Hq, d)), lse=fake((B, Hq, N - 1), torch.float32))
    refused(ea.attn_fwd, q, fake((B, N, Hkv, d), other_device=True), v, o=fake((B, N, Hq, d)))
    refused(ea.attn_fwd, q, k, v, o=fake((B, N, Hq, d), other_device=True))
    refused(ea.attn_fwd_f32o, q, k, v, o=fake((B, N, Hq, d), torch.float32),
            lse=fake((B, Hq, N), torch.float32, other_device=True))


def test_varlen_checks_output_and_lse_shapes():
    total = 40
    q, k, v = fake((total, Hq, d)), fake((total, Hkv, d)), fake((total, Hkv, d))
    cu = fake((3,), torch.int32)
    refused(ea.attn_fwd_varlen, q, k, v, cu, cu, 20, 20, o=fake((total - 1, Hq, d)))
    refused(ea.attn_fwd_varlen, q, k, v, cu, cu, 20, 20, o=fake((total, Hq, d)),
            lse=fake((total, Hq), torch.float32))
    refused(ea.attn_fwd_varlen, q, k, v, fake((3,), torch.int32, other_device=True), cu, 20, 20,
            o=fake((total, Hq, d)))


def test_backward_checks_gradients_lse_and_devices():
    q, k, v = qkv()
    o, do = fake((B, N, Hq, d)), fake((B, N, Hq, d))
    lse = fake((B, Hq, N), torch.float32)
    ws = fake((1 << 20,), torch.uint8)
    refused(ea.attn_bwd, q, k, v, o, fake((B, Hq, N + 1), torch.float32), do, workspace=ws)
    refused(ea.attn_bwd, q, k, v, o, lse, do, dq=fake((B, N, Hq, d // 2)), workspace=ws,
            dk=fake((B, N, Hkv, d)), dv=fake((B, N, Hkv, d)))
    refused(ea.attn_bwd, q, k, v, o, lse, do, dq=fake((B, N, Hq, d)), dk=fake((B, N, Hq, d)),
            dv=fake((B, N, Hkv, d)), workspace=ws)
    refused(ea.attn_bwd, q, k, v, o, lse, fake((B, N, Hq, d), other_device=True),
            dq=fake((B, N, Hq, d)), dk=fake((B, N, Hkv, d)), dv=fake((B, N, Hkv, d)), workspace=ws)
    refused(ea.attn_bwd, q, k, v, o, lse, do, dq=fake((B, N, Hq, d)), dk=fake((B, N, Hkv, d)),
            dv=fake((B, N, Hkv, d)), workspace=fake((1 << 20,), torch.uint8, other_device=True))


def test_merge_checks_output_and_lse_shapes():
    R = 3
    parts, lparts = fake((R, B, N, Hq, d), torch.float32), fake((R, B, Hq, N), torch.float32)
    refused(ea.attn_merge, parts, lparts, o=fake((B, N, Hq - 1, d)))
    refused(ea.attn_merge, parts, lparts, o=fake((B, N, Hq, d)), lse=fake((B, N, Hq), torch.float32))
    refused(ea.attn_merge, parts, fake((R, B, Hq, N), torch.float32, other_device=True),
            o=fake((B, N, Hq, d)))


@pytest.mark.parametrize("entry", ["attn_decode", "attn_decode_noalloc"])
def test_decode_checks_output_lse_seqlens(entry):
    fn = getattr(ea, entry)
    L = 64
    q, kc, vc = fake((B, Hq, d)), fake((B, L, Hkv, d)), fake((B, L, Hkv, d))
    o = fake((B, Hq, d))
    extra = {"workspace": fake((1 << 20,), torch.uint8)} if entry == "attn_decode" else {}
    refused(fn, q, kc, vc, o=fake((B - 1, Hq, d)), **extra)
    refused(fn, q, kc, vc, o=o, lse=fake((B, Hq + 1), torch.float32), **extra)
    refused(fn, q, kc, vc, o=o, seqlens=fake((B - 1,), torch.int32), **extra)
    refused(fn, q, kc, vc, o=o, seqlens=fake((B,), torch.int32, other_device=True), **extra)
    refused(fn, q, fake((B, L, Hkv, d), other_device=True), vc, o=o, **extra)


def test_decode_workspace_on_another_device_is_refused():
    L = 64
    q, kc, vc = fake((B, Hq, d)), fake((B, L, Hkv, d)), fake((B, L, Hkv, d))
    refused(ea.attn_decode, q, kc, vc, o=fake((B, Hq, d)),
            workspace=fake((1 << 20,), torch.uint8, other_device=True))


def test_paged_decode_checks_output_lse_seqlens_table():
    npg, ps, per_seq = 10, 16, 4
    q = fake((B, Hq, d))
    kp, vp = fake((npg, ps, Hkv, d)), fake((npg, ps, Hkv, d))
    bt = fake((B, per_seq), torch.int32)
    ws = fake((1 << 20,), torch.uint8)
    o = fake((B, Hq, d))
    refused(ea.attn_decode_paged, q, kp, vp, bt, o=fake((B, Hq, d + 8)), workspace=ws)
    refused(ea.attn_decode_paged, q, kp, vp, bt, o=o, lse=fake((Hq, B), torch.float32), workspace=ws)
    refused(ea.attn_decode_paged, q, kp, vp, bt, o=o, seqlens=fake((B + 1,), torch.int32),
            workspace=ws)
    refused(ea.attn_decode_paged, q, kp, vp, fake((B, per_seq), torch.int32, other_device=True),
            o=o, workspace=ws)
