"""patch_linear_noalloc: the product without any device allocation in the call.

Callers that cannot allocate device memory while they run (an allocator frozen
after start-up, a memory pool owned by another framework, a thread that may not
call cudaMalloc) use this entry point; its tile schedule lives in a fixed array
of the library's device image instead of memory the library allocates. These
tests call it through the C ABI, two calls in a row on the shared array, and
compare it with patch_linear: bit for bit where both run the same kernel on the
same schedule (M >= 65), and against the CPU oracle within the parity bound of
the other GPU tests where the kernels differ (M <= 64) and for one M >= 65 case.
This file is collected last, so a run that stops at its first failure has
already run every other test.
"""
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


def _noalloc(hsg, lin, X):
    Y = torch.empty((X.shape[0], lin.N), dtype=torch.bfloat16, device="cuda")
    st = hsg.library().patch_linear_noalloc(lin.handle, X.data_ptr(), X.shape[0], Y.data_ptr(),
                                           torch.cuda.current_stream().cuda_stream)
    assert st == 0, hsg.library().patch_last_error().decode()
    return Y


def _oracle_close(p, X, Y):
    """Per element |err| <= 1e-2 * sum_k |x_k w'_k| and relative Frobenius
    error <= 5e-3 against the fp32 oracle (the bound of the parity tests)."""
    import oracle
    Yo, _ = oracle.linear(X.cpu(), p.W.cpu(), p.bits.cpu().numpy())
    Wm = oracle.apply_mask(p.W.cpu(), p.keep.cpu().numpy().astype(np.uint8))
    S = oracle.abs_scale(X.cpu(), Wm)
    Yg = Y.float().cpu().numpy()
    assert np.all(np.abs(Yg - Yo) <= 1e-2 * S + 1e-30)
    assert np.linalg.norm(Yg - Yo) / max(np.linalg.norm(Yo), 1e-30) <= 5e-3


@pytest.mark.parametrize("R,C,frac", [(128, 128, 0.9), (64, 64, 0.5)])
def test_noalloc_matches_patch_linear_twice(hsg, R, C, frac):
    p1 = synth.make_problem(1024, 768, 700, R=R, C=C, frac=frac, seed=1, device="cuda", tag="na1")
    p2 = synth.make_problem(384, 512, 100, R=R, C=C, frac=frac, seed=2, device="cuda", tag="na2")
    l1 = hsg.PackedLinear.pack(p1.W, p1.bits, p1.flags.cpu(), R, C)
    l2 = hsg.PackedLinear.pack(p2.W, p2.bits, p2.flags.cpu(), R, C)
    # calls in a row on the shared schedule array: CTA-pair kernel (M=700),
    # single-CTA kernel (M=100), the first again, then the CUDA-core decode
    # kernel (M=5) and the single-CTA kernel at M=12
    for lin, p, X in ((l1, p1, p1.X), (l2, p2, p2.X), (l1, p1, p1.X)):
        Yn = _noalloc(hsg, lin, X)
        Yr = lin(X)
        torch.cuda.synchronize()
        lin.check()
        assert torch.equal(Yn, Yr)
    _oracle_close(p1, p1.X, Yn)
    for M in (5, 12):
        X = p2.X[:M].contiguous()
        Yn = _noalloc(hsg, l2, X)
        torch.cuda.synchronize()
        _oracle_close(p2, X, Yn)
    l1.free()
    l2.free()


def test_noalloc_rejects_too_many_tiles(hsg):
    p = synth.make_problem(256, 128, 0, frac=0.5, seed=3, device="cuda", tag="na3")
    lin = hsg.PackedLinear.pack(p.W, p.bits, p.flags.cpu())
    buf = torch.empty(16, dtype=torch.bfloat16, device="cuda")  # never read: rejected first
    M = 65537 * 256
    st = hsg.library().patch_linear_noalloc(lin.handle, buf.data_ptr(), M, buf.data_ptr(), None)
    assert st == 2
    msg = hsg.library().patch_last_error().decode()
    assert "65536 output tiles" in msg
    lin.free()
