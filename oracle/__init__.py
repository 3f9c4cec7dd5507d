"""CPU oracle for the PATCH hybrid dense / 2:4 linear layer (test infrastructure).

Only tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may import this package. The product path (``hybrid_sparse_gemm_b200``) never
does, and shares no code with it. The arithmetic lives in ``oracle.c`` (plain
C, built with ``-ffp-contract=off`` so that every fp32 product and sum is
rounded on its own, in the order the C source states); this module only builds
it and marshals numpy arrays.

Definitions followed (see ``oracle.c`` for the full list of readings):
  * mask applied by zeroing pruned weights: model card
    "llama_3.2_1b-PATCH-45Sparse", "How to use" (apply_patch_mask);
  * dense / 2:4 tiles: the same card's method paragraph and the abstract of
    "PATCH: Learnable Tile-level Hybrid Sparsity for LLMs";
  * tile shapes: the card's "Training hyper-parameters" table.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
               "-shared", "-fPIC", "-o", _LIB, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        I = ctypes.c_int
        lib.oracle_f32_to_bf16.argtypes = [ctypes.c_float]
        lib.oracle_f32_to_bf16.restype = ctypes.c_uint16
        lib.oracle_round_bf16.argtypes = [P, I64, P]
        lib.oracle_expand_mask.argtypes = [P, I64, I64, I, P]
        lib.oracle_check_tiles.argtypes = [P, I64, I64, P, I, I, P]
        lib.oracle_check_tiles.restype = I64
        lib.oracle_sparsity.argtypes = [P, I64, I64]
        lib.oracle_sparsity.restype = ctypes.c_double
        lib.oracle_apply_mask.argtypes = [P, P, I64, I64, P]
        lib.oracle_linear_f32.argtypes = [P, I64, I64, P, I64, P, I64, P]
        lib.oracle_abs_scale.argtypes = [P, I64, P, I64, P, I64, P]
        lib.oracle_pack_table.argtypes = [I64, I64, P, I, I, P, P, P]
        lib.oracle_pack_table.restype = I64
        lib.oracle_pair_order.argtypes = [I64, I64, P, I, I, P]
        lib.oracle_pair_order.restype = I
        lib.oracle_pack.argtypes = [P, P, I64, I64, P, P, P, P]
        lib.oracle_pack.restype = I
        lib.oracle_unpack.argtypes = [P, P, P, I64, I64, P]
        lib.oracle_unpack.restype = I
        lib.oracle_unpack_gemm.argtypes = [P, P, P, I64, I64, P]
        lib.oracle_unpack_gemm.restype = I
        _lib = lib
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _u16(a) -> np.ndarray:
    """bf16 data as its uint16 bit pattern (accepts torch bf16 or uint16 numpy)."""
    if isinstance(a, np.ndarray):
        assert a.dtype == np.uint16
        return np.ascontiguousarray(a)
    import torch  # only for the dtype view
    assert a.dtype == torch.bfloat16
    return np.ascontiguousarray(a.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def f32_to_bf16(x: float) -> int:
    return int(_load().oracle_f32_to_bf16(ctypes.c_float(x)))


def round_bf16(y: np.ndarray) -> np.ndarray:
    y = np.ascontiguousarray(y, dtype=np.float32)
    out = np.empty(y.shape, np.uint16)
    _load().oracle_round_bf16(_p(y), y.size, _p(out))
    return out


def bf16_bits_to_f32(u: np.ndarray) -> np.ndarray:
    return (u.astype(np.uint32) << 16).view(np.float32)


def expand_mask(bits: np.ndarray, N: int, K: int, bitorder: int = 0) -> np.ndarray:
    bits = np.ascontiguousarray(bits, dtype=np.uint8)
    assert bits.size >= (N * K + 7) // 8
    keep = np.empty((N, K), np.uint8)
    _load().oracle_expand_mask(_p(bits), N, K, bitorder, _p(keep))
    return keep


def check_tiles(keep: np.ndarray, flags: np.ndarray, R: int, C: int):
    """(bad 2:4 groups, pruned elements inside dense tiles)."""
    N, K = keep.shape
    keep = np.ascontiguousarray(keep, dtype=np.uint8)
    flags = np.ascontiguousarray(flags, dtype=np.uint8)
    stray = ctypes.c_int64(0)
    bad = _load().oracle_check_tiles(_p(keep), N, K, _p(flags), R, C, ctypes.byref(stray))
    return int(bad), int(stray.value)


def sparsity(keep: np.ndarray) -> float:
    keep = np.ascontiguousarray(keep, dtype=np.uint8)
    return float(_load().oracle_sparsity(_p(keep), keep.shape[0], keep.shape[1]))


def apply_mask(W, keep: np.ndarray) -> np.ndarray:
    W = _u16(W)
    N, K = keep.shape
    keep = np.ascontiguousarray(keep, dtype=np.uint8)
    out = np.empty((N, K), np.uint16)
    _load().oracle_apply_mask(_p(W), _p(keep), N, K, _p(out))
    return out


def linear_f32(X, Wm, rows=None) -> np.ndarray:
    """fp32 Y[rows] = X[rows] . Wm^T with an ascending-k fp32 running sum."""
    X = _u16(X)
    Wm = _u16(Wm)
    M, K = X.shape
    N = Wm.shape[0]
    assert Wm.shape[1] == K
    if rows is None:
        r = None
        nrows = M
    else:
        r = np.ascontiguousarray(rows, dtype=np.int64)
        nrows = r.size
    Y = np.empty((nrows, N), np.float32)
    _load().oracle_linear_f32(_p(X), M, K, _p(Wm), N, None if r is None else _p(r), nrows, _p(Y))
    return Y


def abs_scale(X, Wm, rows=None) -> np.ndarray:
    """sum_k |x_k w_k| per output element (fp64)."""
    X = _u16(X)
    Wm = _u16(Wm)
    M, K = X.shape
    N = Wm.shape[0]
    if rows is None:
        r = None
        nrows = M
    else:
        r = np.ascontiguousarray(rows, dtype=np.int64)
        nrows = r.size
    S = np.empty((nrows, N), np.float64)
    _load().oracle_abs_scale(_p(X), K, _p(Wm), N, None if r is None else _p(r), nrows, _p(S))
    return S


def linear(X, W, bits: np.ndarray, bitorder: int = 0, rows=None):
    """The whole path: expand the mask, zero pruned weights, multiply.

    Returns (Y_f32, Y_bf16_bits)."""
    Wu = _u16(W)
    N, K = Wu.shape
    keep = expand_mask(bits, N, K, bitorder)
    Wm = apply_mask(Wu, keep)
    Y = linear_f32(X, Wm, rows)
    return Y, round_bf16(Y)


class Tables:
    """The three uint32 tables of a packed weight (see oracle.c)."""

    def __init__(self, slab, meta, gemm, nbytes):
        self.slab, self.meta, self.gemm, self.nbytes = slab, meta, gemm, nbytes


def pack_table(N: int, K: int, flags, R: int, C: int) -> Tables:
    flags = np.ascontiguousarray(flags, dtype=np.uint8).reshape(-1)
    KB = K // 64
    KC = (KB + 1) // 2
    slab = np.empty((N // 128) * KB, np.uint32)
    meta = np.empty((N // 128) * KC, np.uint32)
    gemm = np.empty((N // 128) * KB, np.uint32)
    total = _load().oracle_pack_table(N, K, _p(flags), R, C, _p(slab), _p(meta), _p(gemm))
    if total < 0:
        raise MemoryError("oracle_pack_table: out of memory")
    return Tables(slab, meta, gemm, int(total))


def pair_order(N: int, K: int, flags, R: int, C: int) -> np.ndarray:
    """Strip order of the CTA-pair view: pair i is strips order[2i], order[2i+1]."""
    flags = np.ascontiguousarray(flags, dtype=np.uint8).reshape(-1)
    order = np.empty(max(N // 128, 1), np.int32)
    if _load().oracle_pair_order(N, K, _p(flags), R, C, _p(order)) != 0:
        raise MemoryError("oracle_pair_order: out of memory")
    return order[:N // 128]


def pack(W, keep: np.ndarray, flags: np.ndarray, R: int, C: int):
    """Independent CPU pack: returns (packed bytes, Tables)."""
    Wu = _u16(W)
    N, K = Wu.shape
    keep = np.ascontiguousarray(keep, dtype=np.uint8)
    t = pack_table(N, K, flags, R, C)
    out = np.zeros(t.nbytes, np.uint8)
    rc = _load().oracle_pack(_p(Wu), _p(keep), N, K, _p(t.slab), _p(t.meta), _p(t.gemm), _p(out))
    if rc != 0:
        raise ValueError("mask is not 2:4 inside a tile flagged 2:4")
    return out, t


def unpack(packed: np.ndarray, t: Tables, N: int, K: int, view: str = "slab") -> np.ndarray:
    """Decode to W' from the per-strip records (view='slab') or from the
    records the tensor-core table points at (view='gemm')."""
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    Wm = np.empty((N, K), np.uint16)
    if view == "slab":
        rc = _load().oracle_unpack(_p(packed), _p(t.slab), _p(t.meta), N, K, _p(Wm))
    else:
        rc = _load().oracle_unpack_gemm(_p(packed), _p(t.gemm), _p(t.meta), N, K, _p(Wm))
    if rc != 0:
        raise ValueError("invalid packed data")
    return Wm
