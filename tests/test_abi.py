"""C-ABI library checks that need no GPU: it loads, exports every symbol the
header declares, rejects bad arguments before touching a device, and its host
slab planner agrees bit for bit with the oracle's restatement of the format."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def hsg():
    import hybrid_sparse_gemm_b200 as m
    return m


def header_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names.update(re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(patch_\w+)\s*\(", src, flags=re.M))
    return sorted(names)


def test_exports_every_header_symbol(hsg):
    names = header_functions()
    assert len(names) >= 12
    lib = hsg.library()
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing
    assert set(names) == set(hsg.EXPORTED)


def test_version(hsg):
    assert hsg.version() == 4


def _pack_status(hsg, W=0x1000, N=256, K=256, bits=0x2000, bitorder=0, flags=None, R=128, C=128):
    lib = hsg.library()
    if flags is None:
        flags = np.zeros(max(1, (N // max(R, 1)) * (K // max(C, 1))), np.uint8)
    h = ctypes.c_void_p()
    st = lib.patch_pack(W, N, K, bits, bitorder, flags.ctypes.data if flags is not False else None,
                        R, C, None, ctypes.byref(h))
    return st, h.value, lib.patch_last_error().decode()


def test_pack_rejects_bad_arguments_without_device(hsg):
    assert _pack_status(hsg, R=96)[0] == 2              # tile shape
    assert _pack_status(hsg, N=200)[0] == 2             # N % 128
    assert _pack_status(hsg, K=96, C=64)[0] == 2        # K % 64
    assert _pack_status(hsg, N=128, R=128, K=192)[0] == 2  # K % C
    assert _pack_status(hsg, N=0)[0] == 2
    assert _pack_status(hsg, W=0)[0] == 1               # NULL
    assert _pack_status(hsg, bits=0)[0] == 1
    assert _pack_status(hsg, flags=False)[0] == 1
    assert _pack_status(hsg, bitorder=2)[0] == 1
    st, h, msg = _pack_status(hsg, W=0x1008)            # not 16-byte aligned
    assert st == 3 and h is None and "aligned" in msg


def test_linear_rejects_bad_arguments(hsg):
    lib = hsg.library()
    assert lib.patch_linear(None, 0x1000, 4, 0x2000, None) == 1
    assert lib.patch_linear_host(None, 0x1000, 4, 0x2000, None) == 1
    assert lib.patch_unpack(None, 0x1000, None) == 1
    assert lib.patch_check(None, None) == 1
    assert lib.patch_copy_packed(None, None, 0, None, 0, None, 0, None, 0) == 1
    assert lib.patch_linear_path(None, 0x1000, 4, 0x2000, 9, None) == 1
    info = hsg.patch_info_t()
    assert lib.patch_info(None, ctypes.byref(info)) == 1
    lib.patch_free(None)  # ignored


def test_pack_without_device_reports_cuda_or_unsupported(hsg):
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    W = torch.zeros(256 * 256 + 8, dtype=torch.bfloat16)
    ptr = W.data_ptr()
    ptr += (-ptr) % 16
    st, h, msg = _pack_status(hsg, W=ptr)
    assert st in (5, 8) and h is None and msg


@pytest.mark.parametrize("R,C", [(128, 128), (128, 64), (64, 128), (64, 64)])
@pytest.mark.parametrize("N,K,frac", [(256, 384, 0.5), (512, 448, 0.9), (128, 64, 1.0),
                                      (384, 1024, 0.0), (1024, 512, 0.3), (640, 320, 0.7)])
def test_plan_matches_oracle_tables(hsg, oracle_lib, R, C, N, K, frac):
    if N % R or K % C:
        pytest.skip("shape not divisible by tile")
    flags = synth.tile_flags(N, K, R, C, frac, "plan").numpy().reshape(-1)
    (slab, meta, gemm), nbytes = hsg.patch_plan(N, K, flags, R, C)
    t = oracle_lib.pack_table(N, K, flags, R, C)
    assert nbytes == t.nbytes
    assert np.array_equal(slab, t.slab)
    assert np.array_equal(meta, t.meta)
    assert np.array_equal(gemm, t.gemm)


@pytest.mark.parametrize("R,C", [(128, 128), (64, 64)])
@pytest.mark.parametrize("N,K,frac,seed", [(1152, 1024, 0.9, 1), (1280, 512, 0.7, 2), (896, 768, 0.5, 3),
                                           (11008, 4096, 0.9, 4), (4096, 4096, 0.6, 5), (640, 256, 1.0, 6),
                                           (384, 2048, 0.0, 7)])
def test_plan_pairs_match_oracle(hsg, oracle_lib, R, C, N, K, frac, seed):
    """The strip pairing of the CTA-pair kernels equals the oracle's
    restatement, and the tables built on it too."""
    flags = synth.tile_flags(N, K, R, C, frac, "pairs", seed).numpy().reshape(-1)
    order = hsg.patch_plan_pairs(N, K, flags, R, C)
    assert np.array_equal(order, oracle_lib.pair_order(N, K, flags, R, C))
    (slab, meta, gemm), nbytes = hsg.patch_plan(N, K, flags, R, C)
    t = oracle_lib.pack_table(N, K, flags, R, C)
    assert nbytes == t.nbytes and np.array_equal(gemm, t.gemm)


def test_plan_checkerboard_and_llama_sizes(hsg, oracle_lib):
    # checkerboard of 64x64 tiles: no 128x64 slab is all-2:4, so nothing compresses
    N, K = 256, 256
    fl = np.indices((N // 64, K // 64)).sum(0) % 2
    (slab, meta, gemm), nbytes = hsg.patch_plan(N, K, fl.astype(np.uint8), 64, 64)
    assert nbytes == N * K * 2 and int((slab & 1).sum()) == 0 and (meta == 0xFFFFFFFF).all()
    # all-2:4 Llama-3.2-1B q projection: 1.125 bytes per weight, no dense images
    (slab, meta, gemm), nbytes = hsg.patch_plan(2048, 2048, np.ones(256, np.uint8), 128, 128)
    assert nbytes == 2048 * 2048 * 9 // 8
    assert np.array_equal(slab, gemm)


def test_plan_errors(hsg):
    with pytest.raises(hsg.PatchError) as e:
        hsg.patch_plan(256, 256, np.zeros(4, np.uint8), 128, 96)
    assert e.value.status == 2
    with pytest.raises(hsg.PatchError) as e:
        hsg.patch_plan(256, 256, np.full(4, 3, np.uint8), 128, 128)
    assert e.value.status == 1
    with pytest.raises(hsg.PatchError) as e:
        hsg.patch_plan_pairs(256, 256, np.zeros(4, np.uint8), 128, 96)
    assert e.value.status == 2


@pytest.mark.parametrize("S", [2048, 2049])
def test_plan_pairs_size_limit(hsg, oracle_lib, S):
    """Up to 2048 strips the pairing follows agreement; above, the fixed
    pairs stay (both sides of the limit, against the oracle)."""
    g = np.random.default_rng(S)
    flags = (g.random((S, 2)) < 0.5).astype(np.uint8).reshape(-1)
    order = hsg.patch_plan_pairs(128 * S, 128, flags, 128, 64)
    assert np.array_equal(order, oracle_lib.pair_order(128 * S, 128, flags, 128, 64))
    assert np.array_equal(order, np.arange(S)) == (S > 2048)


def test_group_and_noalloc_reject_bad_arguments(hsg):
    lib = hsg.library()
    g = ctypes.c_void_p()
    assert lib.patch_linear_noalloc(None, 0x1000, 4, 0x2000, None) == 1
    assert lib.patch_group_create(None, 1, ctypes.byref(g)) == 1 and g.value is None
    nulls = (ctypes.c_void_p * 2)()
    assert lib.patch_group_create(nulls, 2, ctypes.byref(g)) == 1
    assert b"handle 0 is NULL" in lib.patch_last_error()
    assert lib.patch_group_create(nulls, 0, ctypes.byref(g)) == 1
    assert lib.patch_group_create(nulls, 1, None) == 1
    out = ctypes.c_int(-1)
    assert lib.patch_group_path(None, 16, 0, ctypes.byref(out)) == 1 and out.value == -1
    assert lib.patch_group_linear(None, None, 4, None, 0, None) == 1
    lib.patch_group_free(None)  # ignored


def test_last_error_is_the_last_failure_of_this_thread(hsg):
    import threading
    lib = hsg.library()
    seen = []
    t = threading.Thread(target=lambda: seen.append(lib.patch_last_error()))
    t.start()
    t.join()
    assert seen == [b""]                       # a thread with no failed call
    assert lib.patch_linear(None, 0x1000, 4, 0x2000, None) == 1
    msg = lib.patch_last_error()
    assert b"NULL" in msg
    # a successful call leaves the last failure's message in place
    assert hsg.patch_partition_rows(256, 128, np.zeros((2, 1), np.uint8), 1) == [0, 256]
    assert lib.patch_last_error() == msg
    t = threading.Thread(target=lambda: seen.append(lib.patch_last_error()))
    t.start()
    t.join()
    assert seen[-1] == b""                     # other threads do not see it


def test_selftest_without_device(hsg):
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    lib = hsg.library()
    assert lib.patch_selftest_wait(None) in (5, 8)
    assert lib.patch_last_error()
