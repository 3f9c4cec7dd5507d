"""Seeded synthetic inputs for the PATCH hybrid dense / 2:4 linear layer.

This module is shared by the tests, the benchmark and the smoke check; it holds
none of the layer's arithmetic (no mask application, packing or product). It
draws frozen weights, activations, the per-tile dense / 2:4 choice and the
kept set of every 2:4 group, and writes the mask in its released bit-packed
form.

Recipe (the pages ship no weights, masks or data, so every input is drawn):
  * W ~ N(0, 0.02^2), X ~ N(0, 1), drawn in fp32 and rounded to bf16;
  * tile flags: exactly round(f * T) of the T tiles of a matrix are 2:4,
    picked by a seeded permutation; a global fraction can be split
    non-uniformly over several matrices (``split_fraction``);
  * a 2:4 tile keeps the two largest |w| of every group of four consecutive
    k, ties going to the lower k (the "Magnitude" 2:4 rule in the results
    table of the "llama_3.2_1b-PATCH-45Sparse" card);
  * the mask is bit-packed row-major over W[N, K], MSB first by default
    (numpy ``packbits`` order), LSB first on request.
"""
from __future__ import annotations

import hashlib
import math
from dataclasses import dataclass

import torch


def _seed(*parts) -> int:
    h = hashlib.sha256(("/".join(str(p) for p in parts)).encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def generator(device, *parts) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(_seed(*parts))
    return g


def normal_bf16(shape, std: float, device="cpu", *parts) -> torch.Tensor:
    """bf16 tensor with entries N(0, std^2), seeded by ``parts``."""
    g = generator(device, *parts)
    x = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def pick_tiles(n_tiles: int, n_sparse: int, *parts) -> torch.Tensor:
    """uint8 flags over ``n_tiles`` tiles, exactly ``n_sparse`` of them 1 (2:4)."""
    assert 0 <= n_sparse <= n_tiles
    g = generator("cpu", "tiles", *parts)
    perm = torch.randperm(n_tiles, generator=g)
    flags = torch.zeros(n_tiles, dtype=torch.uint8)
    flags[perm[:n_sparse]] = 1
    return flags


def tile_flags(N: int, K: int, R: int, C: int, frac: float, *parts) -> torch.Tensor:
    T = (N // R) * (K // C)
    return pick_tiles(T, int(round(frac * T)), N, K, R, C, *parts).view(N // R, K // C)


def top2_keep(W: torch.Tensor, flags: torch.Tensor, R: int, C: int) -> torch.Tensor:
    """Keep mask (bool, N x K): all-ones in dense tiles, top-2 |w| per group of 4
    along k in 2:4 tiles (ties to the lower index)."""
    N, K = W.shape
    dev = W.device
    a = W.float().abs().view(N, K // 4, 4)
    # rank of element i in its group: how many others beat it (larger, or equal
    # and earlier); the two with rank < 2 are kept.
    ai = a.unsqueeze(-1)          # [..., i, 1]
    aj = a.unsqueeze(-2)          # [..., 1, j]
    idx = torch.arange(4, device=dev)
    earlier = (idx.view(1, 4) < idx.view(4, 1))  # [i, j]: j < i
    beats = (aj > ai) | ((aj == ai) & earlier)
    rank = beats.sum(-1)
    keep24 = (rank < 2).view(N, K)
    f = flags.to(dev).bool().repeat_interleave(R, 0).repeat_interleave(C, 1)
    return torch.where(f, keep24, torch.ones_like(keep24))


def pack_bits(keep: torch.Tensor, bitorder: int = 0) -> torch.Tensor:
    """Row-major bit-packing of a bool N x K mask into ceil(N*K/8) uint8."""
    flat = keep.reshape(-1).to(torch.uint8)
    pad = (-flat.numel()) % 8
    if pad:
        flat = torch.cat([flat, torch.zeros(pad, dtype=torch.uint8, device=flat.device)])
    b = flat.view(-1, 8).to(torch.int32)
    if bitorder == 0:
        w = torch.tensor([128, 64, 32, 16, 8, 4, 2, 1], dtype=torch.int32, device=flat.device)
    else:
        w = torch.tensor([1, 2, 4, 8, 16, 32, 64, 128], dtype=torch.int32, device=flat.device)
    return (b * w).sum(-1).to(torch.uint8)


def split_fraction(tile_counts, target: float, lo: float, hi: float, *parts):
    """Non-uniform per-matrix 2:4 tile counts under one global target.

    Draws f_i ~ U[lo, hi] per matrix, then moves one tile at a time (largest
    remainder first) until the tile-weighted total equals round(target * T)
    exactly. Counts stay within each matrix's tile count."""
    g = generator("cpu", "split", *parts)
    n = len(tile_counts)
    f = lo + (hi - lo) * torch.rand(n, generator=g, dtype=torch.float64)
    T = sum(tile_counts)
    want = int(round(target * T))
    raw = [float(f[i]) * tile_counts[i] for i in range(n)]
    cnt = [min(tile_counts[i], max(0, int(math.floor(raw[i])))) for i in range(n)]
    order_up = sorted(range(n), key=lambda i: -(raw[i] - math.floor(raw[i])))
    guard = 0
    while sum(cnt) != want and guard < 10 * T + 10:
        guard += 1
        if sum(cnt) < want:
            for i in order_up + list(range(n)):
                if cnt[i] < tile_counts[i]:
                    cnt[i] += 1
                    break
        else:
            for i in list(reversed(order_up)) + list(range(n)):
                if cnt[i] > 0:
                    cnt[i] -= 1
                    break
    assert sum(cnt) == want
    return cnt


@dataclass
class Linear:
    name: str
    N: int
    K: int


def llama32_1b():
    """Linear shapes of one Llama-3.2-1B layer (hidden 2048, kv 512, ffn 8192)."""
    return [Linear("q", 2048, 2048), Linear("k", 512, 2048), Linear("v", 512, 2048),
            Linear("o", 2048, 2048), Linear("gate", 8192, 2048), Linear("up", 8192, 2048),
            Linear("down", 2048, 8192)]


def llama2_7b():
    return [Linear("q", 4096, 4096), Linear("k", 4096, 4096), Linear("v", 4096, 4096),
            Linear("o", 4096, 4096), Linear("gate", 11008, 4096), Linear("up", 11008, 4096),
            Linear("down", 4096, 11008)]


def llama2_13b():
    return [Linear("q", 5120, 5120), Linear("k", 5120, 5120), Linear("v", 5120, 5120),
            Linear("o", 5120, 5120), Linear("gate", 13824, 5120), Linear("up", 13824, 5120),
            Linear("down", 5120, 13824)]


@dataclass
class Problem:
    """One linear layer's inputs: W bf16 [N,K], flags uint8 [N/R, K/C],
    keep bool [N,K], bits uint8, tile shape, and X bf16 [M,K]."""
    W: torch.Tensor
    flags: torch.Tensor
    keep: torch.Tensor
    bits: torch.Tensor
    R: int
    C: int
    X: torch.Tensor | None = None
    bitorder: int = 0


def make_problem(N, K, M, R=128, C=128, frac=0.5, n_sparse=None, seed=0, device="cpu",
                 bitorder=0, tag="p", w_std=0.02) -> Problem:
    W = normal_bf16((N, K), w_std, device, tag, "W", seed, N, K)
    T = (N // R) * (K // C)
    if n_sparse is None:
        n_sparse = int(round(frac * T))
    flags = pick_tiles(T, n_sparse, tag, seed, N, K, R, C).view(N // R, K // C)
    keep = top2_keep(W, flags, R, C)
    bits = pack_bits(keep, bitorder)
    X = normal_bf16((M, K), 1.0, device, tag, "X", seed, M, K) if M > 0 else \
        torch.empty((0, K), dtype=torch.bfloat16, device=device)
    return Problem(W=W, flags=flags, keep=keep, bits=bits, R=R, C=C, X=X, bitorder=bitorder)
