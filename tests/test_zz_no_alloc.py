"""patch_linear_noalloc: the product without any device allocation in the call.

Callers that cannot allocate device memory while they run (a frozen allocator,
a pool owned by another framework) use this entry point; its tile schedule
lives in a fixed array of the library's device image instead of memory the
library allocates. These tests call it through the C ABI and compare it with
patch_linear, within the parity tolerance of the other GPU tests, on two calls
in a row (the shared array must not keep anything from the previous call that
changes the result).
"""
import ctypes

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hsg():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import hybrid_sparse_gemm_b200 as m
    return m


def _close(a, b):
    a, b = a.float(), b.float()
    scale = b.abs().max().item() + 1e-30
    assert torch.isfinite(a).all()
    assert (a - b).abs().max().item() <= 1e-2 * scale
    assert ((a - b).norm() / (b.norm() + 1e-30)).item() <= 5e-3


def _noalloc(hsg, lin, X):
    Y = torch.empty((X.shape[0], lin.N), dtype=torch.bfloat16, device="cuda")
    st = hsg.library().patch_linear_noalloc(lin.handle, X.data_ptr(), X.shape[0], Y.data_ptr(),
                                           torch.cuda.current_stream().cuda_stream)
    assert st == 0, hsg.library().patch_last_error().decode()
    return Y


@pytest.mark.parametrize("R,C,frac", [(128, 128, 0.9), (64, 64, 0.5)])
def test_noalloc_matches_patch_linear_twice(hsg, R, C, frac):
    p1 = synth.make_problem(1024, 768, 700, R=R, C=C, frac=frac, seed=1, device="cuda", tag="na1")
    p2 = synth.make_problem(384, 512, 100, R=R, C=C, frac=frac, seed=2, device="cuda", tag="na2")
    l1 = hsg.PackedLinear.pack(p1.W, p1.bits, p1.flags.cpu(), R, C)
    l2 = hsg.PackedLinear.pack(p2.W, p2.bits, p2.flags.cpu(), R, C)
    # two calls in a row on the shared schedule array: CTA-pair kernel (M=700),
    # then single-CTA kernel (M=100), then the first again, then decode (M=5)
    for lin, X in ((l1, p1.X), (l2, p2.X), (l1, p1.X), (l2, p2.X[:5].contiguous())):
        Yn = _noalloc(hsg, lin, X)
        Yr = lin(X)
        torch.cuda.synchronize()
        lin.check()
        _close(Yn, Yr)
    l1.free()
    l2.free()


def test_noalloc_rejects_too_many_tiles(hsg):
    p = synth.make_problem(256, 128, 0, frac=0.5, seed=3, device="cuda", tag="na3")
    lin = hsg.PackedLinear.pack(p.W, p.bits, p.flags.cpu())
    buf = torch.empty(16, dtype=torch.bfloat16, device="cuda")  # never read: rejected first
    M = 65537 * 256
    st = hsg.library().patch_linear_noalloc(lin.handle, buf.data_ptr(), M, buf.data_ptr(), None)
    assert st == 2
    assert "65536" in hsg.library().patch_last_error().decode()
    lin.free()
