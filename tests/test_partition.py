"""Output-feature (tensor-parallel) split on the CPU: the cost-balanced row
partition, the shard slicing, and the single-rank exchange.

The partition is pinned against brute force: every contiguous aligned split
of a small weight is scored with a cost written here from the definition (per
256-row strip pair and 64-column slab, dense 1 and 2:4-in-both-strips 1/2,
plus 1 per pair for its epilogue), and the library's split must reach the
smallest largest-shard cost.
"""
import itertools

import numpy as np
import pytest
import torch

import synth

import hybrid_sparse_gemm_b200 as hsg
from hybrid_sparse_gemm_b200 import dist


def pair_costs(flags, N, K, R, C):
    """Cost of every strip pair in half dense slabs (integers)."""
    f = np.asarray(flags).reshape(N // R, K // C)
    S = N // 128

    def slab_sparse(s, b):
        return all(f[r, (b * 64) // C] for r in range(s * 128 // R, (s + 1) * 128 // R))

    costs = []
    for q in range((S + 1) // 2):
        strips = [2 * q, 2 * q + 1] if 2 * q + 1 < S else [2 * q]
        costs.append(2 + sum(1 if all(slab_sparse(s, b) for s in strips) else 2 for b in range(K // 64)))
    return costs


def split_cost(costs, bounds, align):
    out = []
    for r in range(len(bounds) - 1):
        q0, q1 = bounds[r] // 256, -(-bounds[r + 1] // 256)
        assert bounds[r] % align == 0 or bounds[r] == bounds[-1]
        out.append(sum(costs[q0:q1]))
    return max(out)


def brute_force(costs, parts, align):
    per = align // 256
    units = [sum(costs[i:i + per]) for i in range(0, len(costs), per)]
    best = None
    for cuts in itertools.combinations_with_replacement(range(len(units) + 1), parts - 1):
        edges = (0,) + cuts + (len(units),)
        worst = max(sum(units[edges[i]:edges[i + 1]]) for i in range(parts))
        best = worst if best is None else min(best, worst)
    return best, len(units)


CASES = [(N, K, R, C) for N in (128, 384, 1024, 1536, 2304) for K in (128, 512)
         for R, C in ((128, 128), (128, 64), (64, 128), (64, 64))]


@pytest.mark.parametrize("N,K,R,C", CASES)
@pytest.mark.parametrize("parts", [1, 2, 3, 5])
def test_partition_is_optimal_and_well_formed(N, K, R, C, parts):
    for seed, frac in ((0, 0.3), (1, 0.8), (2, 1.0)):
        T = (N // R) * (K // C)
        flags = synth.pick_tiles(T, int(round(frac * T)), "part", seed, N, K, R, C).numpy()
        costs = pair_costs(flags, N, K, R, C)
        for align in (256, 512):
            b = hsg.patch_partition_rows(N, K, flags, parts, R, C, align)
            assert len(b) == parts + 1 and b[0] == 0 and b[-1] == N
            assert all(x <= y for x, y in zip(b, b[1:]))
            assert all(x % align == 0 or x == N for x in b)
            best, units = brute_force(costs, parts, align)
            assert split_cost(costs, b, align) == best, (b, costs)
            widths = [y - x for x, y in zip(b, b[1:])]
            nonempty = [w > 0 for w in widths]
            assert sum(nonempty) == min(parts, units)
            assert nonempty == sorted(nonempty, reverse=True)  # only trailing shards are empty


def test_partition_follows_cost_not_row_count():
    # the first two strip pairs dense, the other six 2:4: the dense rows get
    # a shard of their own size, not half the rows
    N = K = 2048
    f = np.ones((16, 16), np.uint8)
    f[:4] = 0
    assert hsg.patch_partition_rows(N, K, f, 2) == [0, 768, 2048]
    assert hsg.patch_partition_rows(N, K, f, 3) == [0, 512, 1280, 2048]
    assert hsg.patch_partition_rows(N, K, np.zeros((16, 16), np.uint8), 4) == [0, 512, 1024, 1536, 2048]


def test_partition_errors():
    f = np.zeros((4, 4), np.uint8)
    for parts, align, status in ((0, 256, 1), (2, 128, 1), (2, 0, 1), (2, 384, 1)):
        with pytest.raises(hsg.PatchError) as e:
            hsg.patch_partition_rows(512, 512, f, parts, align_rows=align)
        assert e.value.status == status
    with pytest.raises(hsg.PatchError) as e:
        hsg.patch_partition_rows(500, 512, np.zeros(16, np.uint8), 2)
    assert e.value.status == 2
    bad = f.copy()
    bad[1, 2] = 2
    with pytest.raises(hsg.PatchError) as e:
        hsg.patch_partition_rows(512, 512, bad, 2)
    assert e.value.status == 1
    with pytest.raises(ValueError):
        hsg.patch_partition_rows(512, 512, np.zeros(15, np.uint8), 2)


@pytest.mark.parametrize("R,C", [(128, 128), (64, 64)])
def test_shard_rows_cut_whole_rows(oracle_lib, R, C):
    N, K = 1280, 256
    p = synth.make_problem(N, K, 0, R=R, C=C, frac=0.6, seed=4)
    bounds = hsg.patch_partition_rows(N, K, p.flags.numpy(), 3, R, C)
    keep = p.keep.numpy().astype(np.uint8)
    Ws, Bs, Fs = [], [], []
    for r in range(3):
        W, bits, flags = dist.shard_rows(p.W, p.bits, p.flags, R, bounds, r)
        n0, n1 = bounds[r], bounds[r + 1]
        assert W.shape == (n1 - n0, K) and flags.shape == ((n1 - n0) // R, K // C)
        # the byte range decodes to exactly this shard's keep bits
        assert np.array_equal(oracle_lib.expand_mask(bits.numpy(), n1 - n0, K), keep[n0:n1])
        Ws.append(W)
        Bs.append(bits)
        Fs.append(flags)
    assert torch.equal(torch.cat(Ws), p.W) and torch.equal(torch.cat(Bs), p.bits.reshape(-1))
    assert torch.equal(torch.cat(Fs), p.flags.reshape(N // R, -1))
    with pytest.raises(ValueError):
        dist.shard_rows(p.W, p.bits, p.flags, R, [0, 100, N], 0)


def test_single_rank_exchange_is_the_local_block():
    bounds = [0, 384]
    send, y = dist.local_buffer(5, bounds, 0, "cpu")
    y.copy_(torch.arange(5 * 384, dtype=torch.float32).view(5, 384).to(torch.bfloat16))
    out = dist.gather_columns(send, 5, bounds, active=False)
    assert torch.equal(out, y)


def test_exchange_over_several_ranks_needs_a_group():
    send, _ = dist.local_buffer(2, [0, 256, 512], 0, "cpu")
    with pytest.raises(ValueError):
        dist.gather_columns(send, 2, [0, 256, 512], active=False)
