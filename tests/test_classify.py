"""Tile flags derived from a bit-packed keep mask (patch_classify_tiles), on
the CPU.

Pinned two ways: the seeded problems are built from their flags (dense tiles
keep everything, 2:4 tiles keep the top two of every four), so the flags must
come back exactly; and random masks whose tiles mix every case (all kept,
valid 2:4, one group off by one, none kept, arbitrary) are classified here
from the unpacked bits by the definition and must agree tile for tile.
"""
import numpy as np
import pytest

import synth

import hybrid_sparse_gemm_b200 as hsg


@pytest.mark.parametrize("R,C", [(128, 128), (128, 64), (64, 128), (64, 64)])
@pytest.mark.parametrize("frac", [0.0, 0.5, 1.0])
@pytest.mark.parametrize("bitorder", [0, 1])
def test_flags_of_generated_problems_come_back(R, C, frac, bitorder):
    N, K = 384, 512
    p = synth.make_problem(N, K, 0, R=R, C=C, frac=frac, seed=5, bitorder=bitorder, tag="cls")
    flags, stray = hsg.patch_classify_tiles(p.bits, N, K, R, C)
    assert np.array_equal(flags, p.flags.numpy().reshape(N // R, K // C))
    assert stray == 0


def _random_mask(N, K, R, C, rng):
    keep = np.zeros((N, K), np.uint8)
    kinds = rng.integers(0, 6, size=(N // R, K // C))
    for tr in range(N // R):
        for tc in range(K // C):
            t = keep[tr * R:(tr + 1) * R, tc * C:(tc + 1) * C]
            kind = kinds[tr, tc]
            if kind == 0:
                t[:] = 1
            elif kind in (1, 2, 3):
                g = t.reshape(R, C // 4, 4)
                for r in range(R):
                    for j in range(C // 4):
                        g[r, j, rng.choice(4, 2, replace=False)] = 1
                if kind == 2:   # one group keeps three
                    g[rng.integers(R), rng.integers(C // 4)] = [1, 1, 1, 0]
                if kind == 3:   # one group keeps one
                    g[rng.integers(R), rng.integers(C // 4)] = [0, 0, 1, 0]
            elif kind == 4:
                pass            # nothing kept
            else:
                t[:] = rng.integers(0, 2, size=t.shape)
    return keep


def _classify_by_definition(keep, R, C):
    N, K = keep.shape
    flags = np.zeros((N // R, K // C), np.uint8)
    stray = 0
    for tr in range(N // R):
        for tc in range(K // C):
            t = keep[tr * R:(tr + 1) * R, tc * C:(tc + 1) * C]
            sparse = bool((t.reshape(R, C // 4, 4).sum(-1) == 2).all())
            flags[tr, tc] = sparse
            stray += (not sparse) and not t.all()
    return flags, stray


@pytest.mark.parametrize("R,C", [(128, 128), (64, 64), (64, 128)])
@pytest.mark.parametrize("bitorder", ["big", "little"])
def test_random_masks_match_the_definition(R, C, bitorder):
    rng = np.random.default_rng(17 + R + C)
    N, K = 256, 384 if C == 128 else 320
    keep = _random_mask(N, K, R, C, rng)
    bits = np.packbits(keep.reshape(-1), bitorder=bitorder)
    flags, stray = hsg.patch_classify_tiles(bits, N, K, R, C)
    want_flags, want_stray = _classify_by_definition(keep, R, C)
    assert np.array_equal(flags, want_flags)
    assert stray == want_stray
    assert want_flags.any() and not want_flags.all() and want_stray > 0  # the mix covers every branch


def test_classify_errors():
    with pytest.raises(hsg.PatchError) as e:
        hsg.patch_classify_tiles(np.zeros(100 * 128 // 8, np.uint8), 100, 128)
    assert e.value.status == 2
    with pytest.raises(ValueError):
        hsg.patch_classify_tiles(np.zeros(10, np.uint8), 128, 128)
