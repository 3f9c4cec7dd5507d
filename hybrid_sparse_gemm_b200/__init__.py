"""Python binding of the sm_100a hybrid dense / 2:4 linear layer (PATCH).

Argument marshalling only: every step of the layer runs in the CUDA kernels of
``libpatch_hybrid.so`` (the C ABI declared in ``include/patch_hybrid.h``).
PyTorch supplies device memory and streams. If the library is missing this
module raises on import; there is no fallback.

    import hybrid_sparse_gemm_b200 as hsg
    lin = hsg.PackedLinear.pack(W, mask_bits, tile_flags, tile_rows=128, tile_cols=128)
    Y = lin(X)                       # Y = X @ (W * mask).T, bf16
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("PATCH_HYBRID_LIB") or os.path.join(_HERE, "libpatch_hybrid.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m hybrid_sparse_gemm_b200.build`")

_lib = ctypes.CDLL(LIB_PATH)

PATCH_OK = 0
STATUS_NAMES = {0: "PATCH_OK", 1: "PATCH_ERR_ARG", 2: "PATCH_ERR_SHAPE", 3: "PATCH_ERR_ALIGN",
                4: "PATCH_ERR_MASK", 5: "PATCH_ERR_CUDA", 6: "PATCH_ERR_TIMEOUT",
                7: "PATCH_ERR_NOMEM", 8: "PATCH_ERR_UNSUPPORTED"}
PATH_AUTO, PATH_GEMM, PATH_GEMV, PATH_GEMM_SINGLE, PATH_GEMM_PAIR, PATH_GEMV_SIMT, PATH_GEMM_WIDE = 0, 1, 2, 3, 4, 5, 6
PATH_GEMM_WIDE_24 = 7

EXPORTED = ["patch_pack", "patch_linear", "patch_linear_path", "patch_linear_host", "patch_unpack",
            "patch_info", "patch_copy_packed", "patch_check", "patch_free", "patch_last_error",
            "patch_version", "patch_plan", "patch_linear_noalloc", "patch_group_create",
            "patch_group_linear", "patch_group_path", "patch_group_free", "patch_selftest_wait",
            "patch_partition_rows", "patch_classify_tiles", "patch_group_linear_host", "patch_plan_pairs"]


class patch_info_t(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int64), ("K", ctypes.c_int64),
                ("tile_rows", ctypes.c_int32), ("tile_cols", ctypes.c_int32),
                ("tiles_total", ctypes.c_int64), ("tiles_sparse", ctypes.c_int64),
                ("slabs_total", ctypes.c_int64), ("slabs_sparse", ctypes.c_int64),
                ("slabs_pair_sparse", ctypes.c_int64), ("meta_blocks", ctypes.c_int64),
                ("dense_images", ctypes.c_int64), ("packed_bytes", ctypes.c_int64), ("pruned", ctypes.c_int64),
                ("stray_zeros", ctypes.c_int64), ("sparsity", ctypes.c_double)]


_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I = ctypes.c_int
_lib.patch_pack.argtypes = [_P, _I64, _I64, _P, _I, _P, _I, _I, _P, ctypes.POINTER(_P)]
_lib.patch_linear.argtypes = [_P, _P, _I64, _P, _P]
_lib.patch_linear_path.argtypes = [_P, _P, _I64, _P, _I, _P]
_lib.patch_linear_host.argtypes = [_P, _P, _I64, _P, _P]
_lib.patch_linear_noalloc.argtypes = [_P, _P, _I64, _P, _P]
_lib.patch_group_create.argtypes = [_P, _I, ctypes.POINTER(_P)]
_lib.patch_group_linear.argtypes = [_P, _P, _I64, _P, _I, _P]
_lib.patch_group_linear_host.argtypes = [_P, _P, _I64, _P, _I, _P]
_lib.patch_group_path.argtypes = [_P, _I64, _I, ctypes.POINTER(_I)]
_lib.patch_group_free.argtypes = [_P]
_lib.patch_selftest_wait.argtypes = [_P]
_lib.patch_group_free.restype = None
_lib.patch_unpack.argtypes = [_P, _P, _P]
_lib.patch_info.argtypes = [_P, ctypes.POINTER(patch_info_t)]
_lib.patch_copy_packed.argtypes = [_P, _P, _I64, _P, _I64, _P, _I64, _P, _I64]
_lib.patch_check.argtypes = [_P, _P]
_lib.patch_plan.argtypes = [_I64, _I64, _P, _I, _I, _P, _P, _P, ctypes.POINTER(_I64)]
_lib.patch_plan_pairs.argtypes = [_I64, _I64, _P, _I, _I, _P]
_lib.patch_partition_rows.argtypes = [_I64, _I64, _P, _I, _I, _I, _I64, _P]
_lib.patch_classify_tiles.argtypes = [_P, _I64, _I64, _I, _I, _P, ctypes.POINTER(_I64)]
_lib.patch_free.argtypes = [_P]
_lib.patch_free.restype = None
_lib.patch_last_error.restype = ctypes.c_char_p
_lib.patch_version.restype = ctypes.c_int
for _n in ["patch_pack", "patch_linear", "patch_linear_path", "patch_linear_host", "patch_unpack",
           "patch_info", "patch_copy_packed", "patch_check", "patch_plan", "patch_linear_noalloc",
           "patch_group_create", "patch_group_linear", "patch_partition_rows", "patch_classify_tiles",
           "patch_group_linear_host", "patch_plan_pairs"]:
    getattr(_lib, _n).restype = ctypes.c_int


class PatchError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


def _check(status: int):
    if status != PATCH_OK:
        raise PatchError(status, _lib.patch_last_error().decode())


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def library() -> ctypes.CDLL:
    return _lib


def version() -> int:
    return _lib.patch_version()


# ---- thin functions with the C ABI's names -----------------------------------

def _table_sizes(N: int, K: int):
    S, KB = N // 128, K // 64
    return S * KB, S * ((KB + 1) // 2), S * KB


def patch_plan(N: int, K: int, tile_flags, tile_rows: int = 128, tile_cols: int = 128):
    """Host-only: ((slab, meta, gemm) tables as uint32 numpy arrays, packed byte count)."""
    import numpy as np
    flags = np.ascontiguousarray(np.asarray(tile_flags, dtype=np.uint8).reshape(-1))
    ok = N > 0 and K > 0 and N % 128 == 0 and K % 64 == 0
    ns, nm, ng = _table_sizes(N, K) if ok else (0, 0, 0)
    slab, meta, gemm = (np.zeros(max(n, 1), np.uint32) for n in (ns, nm, ng))
    nbytes = _I64(0)
    _check(_lib.patch_plan(N, K, flags.ctypes.data, tile_rows, tile_cols, slab.ctypes.data,
                           meta.ctypes.data, gemm.ctypes.data, ctypes.byref(nbytes)))
    return (slab[:ns], meta[:nm], gemm[:ng]), int(nbytes.value)


def patch_plan_pairs(N: int, K: int, tile_flags, tile_rows: int = 128, tile_cols: int = 128):
    """Host-only: the strip order of the CTA-pair kernels as an int32 numpy
    array of N/128 entries (pair i = strips order[2i], order[2i+1])."""
    import numpy as np
    flags = np.ascontiguousarray(np.asarray(tile_flags, dtype=np.uint8).reshape(-1))
    S = N // 128 if N > 0 and N % 128 == 0 else 0
    order = np.zeros(max(S, 1), np.int32)
    _check(_lib.patch_plan_pairs(N, K, flags.ctypes.data, tile_rows, tile_cols, order.ctypes.data))
    return order[:S]


def patch_classify_tiles(mask_bits, N: int, K: int, tile_rows: int = 128, tile_cols: int = 128):
    """Host-only: (tile flags as a uint8 numpy array [N/tile_rows, K/tile_cols],
    number of dense tiles that prune some weight) for a bit-packed mask."""
    import numpy as np
    bits = mask_bits.cpu().numpy() if isinstance(mask_bits, torch.Tensor) else np.asarray(mask_bits)
    bits = np.ascontiguousarray(bits.reshape(-1), dtype=np.uint8)
    if bits.size != (N * K + 7) // 8:
        raise ValueError(f"mask_bits has {bits.size} bytes, a {N}x{K} mask needs {(N * K + 7) // 8}")
    ok = tile_rows > 0 and tile_cols > 0 and N > 0 and K > 0 and N % tile_rows == 0 and K % tile_cols == 0
    flags = np.zeros(max((N // tile_rows) * (K // tile_cols) if ok else 1, 1), np.uint8)
    stray = _I64(0)
    _check(_lib.patch_classify_tiles(bits.ctypes.data, N, K, tile_rows, tile_cols, flags.ctypes.data,
                                     ctypes.byref(stray)))
    return flags.reshape(N // tile_rows, K // tile_cols), int(stray.value)


def patch_partition_rows(N: int, K: int, tile_flags, parts: int, tile_rows: int = 128, tile_cols: int = 128,
                         align_rows: int = 256) -> list[int]:
    """Host-only: parts + 1 row bounds of a cost-balanced contiguous split of W."""
    import numpy as np
    flags = np.ascontiguousarray(np.asarray(tile_flags, dtype=np.uint8).reshape(-1))
    if tile_rows > 0 and tile_cols > 0 and N % tile_rows == 0 and K % tile_cols == 0 and N > 0 and K > 0:
        if flags.size != (N // tile_rows) * (K // tile_cols):
            raise ValueError(f"tile_flags has {flags.size} entries, the {N}x{K} weight has "
                             f"{(N // tile_rows) * (K // tile_cols)} tiles")
    bounds = np.zeros(max(parts, 0) + 1, np.int64)
    _check(_lib.patch_partition_rows(N, K, flags.ctypes.data, tile_rows, tile_cols, parts, align_rows,
                                     bounds.ctypes.data))
    return [int(b) for b in bounds]


def patch_pack(W: torch.Tensor, mask_bits: torch.Tensor, tile_flags, tile_rows: int = 128,
               tile_cols: int = 128, bitorder: int = 0, stream=None) -> int:
    """Returns an opaque handle (int). W bf16 [N,K] and mask_bits uint8 on the
    device; tile_flags uint8 on the host (any array-like)."""
    assert W.is_cuda and W.dtype == torch.bfloat16 and W.dim() == 2 and W.is_contiguous()
    assert mask_bits.is_cuda and mask_bits.dtype == torch.uint8 and mask_bits.is_contiguous()
    flags = torch.as_tensor(tile_flags, dtype=torch.uint8).reshape(-1).contiguous().cpu()
    N, K = W.shape
    h = _P()
    _check(_lib.patch_pack(W.data_ptr(), N, K, mask_bits.data_ptr(), bitorder, flags.data_ptr(),
                           tile_rows, tile_cols, _stream(stream), ctypes.byref(h)))
    return h.value


def patch_linear_path(h: int, X: torch.Tensor, Y: torch.Tensor, path: int = PATH_AUTO, stream=None):
    _check(_lib.patch_linear_path(h, X.data_ptr(), X.shape[0], Y.data_ptr(), path, _stream(stream)))


def patch_linear(h: int, X: torch.Tensor, Y: torch.Tensor, stream=None):
    _check(_lib.patch_linear(h, X.data_ptr(), X.shape[0], Y.data_ptr(), _stream(stream)))


def patch_linear_noalloc(h: int, X: torch.Tensor, Y: torch.Tensor, stream=None):
    """patch_linear that allocates no device memory (see the header)."""
    _check(_lib.patch_linear_noalloc(h, X.data_ptr(), X.shape[0], Y.data_ptr(), _stream(stream)))


def patch_linear_host(h: int, X: torch.Tensor, Y: torch.Tensor, stream=None):
    """X, Y are CPU tensors (pinned for speed); synchronous."""
    assert not X.is_cuda and not Y.is_cuda
    _check(_lib.patch_linear_host(h, X.data_ptr(), X.shape[0], Y.data_ptr(), _stream(stream)))


def patch_unpack(h: int, out: torch.Tensor, stream=None):
    _check(_lib.patch_unpack(h, out.data_ptr(), _stream(stream)))


def patch_info(h: int) -> patch_info_t:
    info = patch_info_t()
    _check(_lib.patch_info(h, ctypes.byref(info)))
    return info


def patch_copy_packed(h: int):
    """(packed bytes as a uint8 numpy array, (slab, meta, gemm) uint32 tables)."""
    import numpy as np
    info = patch_info(h)
    ns, nm, ng = _table_sizes(int(info.N), int(info.K))
    packed = np.empty(int(info.packed_bytes), np.uint8)
    slab, meta, gemm = np.empty(ns, np.uint32), np.empty(nm, np.uint32), np.empty(ng, np.uint32)
    _check(_lib.patch_copy_packed(h, packed.ctypes.data, packed.size, slab.ctypes.data, ns,
                                  meta.ctypes.data, nm, gemm.ctypes.data, ng))
    return packed, (slab, meta, gemm)


def patch_check(h: int, stream=None):
    _check(_lib.patch_check(h, _stream(stream)))


def patch_free(h: int):
    _lib.patch_free(h)


class LinearGroup:
    """Several packed linears run with one launch (they share M)."""

    def __init__(self, linears):
        self.linears = list(linears)
        arr = (_P * len(self.linears))(*[l.handle for l in self.linears])
        g = _P()
        _check(_lib.patch_group_create(arr, len(self.linears), ctypes.byref(g)))
        self.handle = g.value

    def __call__(self, Xs, outs=None, path: int = PATH_AUTO, stream=None):
        n = len(self.linears)
        assert len(Xs) == n
        M = Xs[0].shape[0]
        if outs is None:
            outs = [torch.empty((M, l.N), dtype=torch.bfloat16, device=Xs[0].device) for l in self.linears]
        xs = (_P * n)(*[x.data_ptr() for x in Xs])
        ys = (_P * n)(*[y.data_ptr() for y in outs])
        _check(_lib.patch_group_linear(self.handle, xs, M, ys, path, _stream(stream)))
        return outs

    def host(self, Xs, outs=None, path: int = PATH_AUTO, stream=None, sync: bool = True):
        """Host tensors in and out (pinned for overlapped copies). With
        sync=False the call only enqueues: the outputs are complete once
        `stream` is."""
        n = len(self.linears)
        assert len(Xs) == n and all(not x.is_cuda for x in Xs)
        M = Xs[0].shape[0]
        if outs is None:
            outs = [torch.empty((M, l.N), dtype=torch.bfloat16, pin_memory=True) for l in self.linears]
        xs = (_P * n)(*[x.data_ptr() for x in Xs])
        ys = (_P * n)(*[y.data_ptr() for y in outs])
        _check(_lib.patch_group_linear_host(self.handle, xs, M, ys, path, _stream(stream)))
        if sync:
            torch.cuda.synchronize()
        return outs

    def path(self, M: int, path: int = PATH_AUTO) -> int:
        """The explicit path a call with this M and requested path would run."""
        out = _I()
        _check(_lib.patch_group_path(self.handle, M, path, ctypes.byref(out)))
        return out.value

    def free(self):
        if self.handle:
            _lib.patch_group_free(self.handle)
            self.handle = 0

    def __del__(self):
        try:
            self.free()
        except Exception:
            pass


# ---- object wrapper -----------------------------------------------------------

class PackedLinear:
    """A frozen weight packed as dense / 2:4 slabs; calling it runs the layer."""

    def __init__(self, handle: int, N: int, K: int):
        self.handle = handle
        self.N = N
        self.K = K

    @classmethod
    def pack(cls, W, mask_bits, tile_flags, tile_rows=128, tile_cols=128, bitorder=0, stream=None):
        h = patch_pack(W, mask_bits, tile_flags, tile_rows, tile_cols, bitorder, stream)
        return cls(h, W.shape[0], W.shape[1])

    def __call__(self, X: torch.Tensor, out: torch.Tensor | None = None, path: int = PATH_AUTO,
                 stream=None) -> torch.Tensor:
        assert X.is_cuda and X.dtype == torch.bfloat16 and X.dim() == 2 and X.shape[1] == self.K
        assert X.is_contiguous()
        if out is None:
            out = torch.empty((X.shape[0], self.N), dtype=torch.bfloat16, device=X.device)
        patch_linear_path(self.handle, X, out, path, stream)
        return out

    def host(self, X: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        if out is None:
            out = torch.empty((X.shape[0], self.N), dtype=torch.bfloat16, pin_memory=True)
        patch_linear_host(self.handle, X, out, stream)
        return out

    def unpack(self, stream=None) -> torch.Tensor:
        out = torch.empty((self.N, self.K), dtype=torch.bfloat16, device="cuda")
        patch_unpack(self.handle, out, stream)
        return out

    def info(self) -> patch_info_t:
        return patch_info(self.handle)

    def packed(self):
        return patch_copy_packed(self.handle)

    def check(self, stream=None):
        patch_check(self.handle, stream)

    def free(self):
        if self.handle:
            patch_free(self.handle)
            self.handle = 0

    def __del__(self):
        try:
            self.free()
        except Exception:
            pass
