"""Parity of the CUDA path with the CPU oracle, through the C ABI (needs a B200).

Bar: the packed bytes and slab table are bit-exact; the product is within
|err| <= 1e-2 * sum_k |x_k w_k| per element and relative Frobenius error
<= 5e-3 of the oracle's fp32 result. Full-size workloads are checked on a
seeded sample of token rows (rows of the product are independent, so the
oracle computes exactly those rows), always including the first and last row.
"""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

TOL_ELEM = 1e-2
TOL_FRO = 5e-3


@pytest.fixture(scope="module")
def hsg():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import hybrid_sparse_gemm_b200 as m
    return m


def sample_rows(M, n=128, seed=0):
    if M <= n:
        return np.arange(M)
    g = np.random.default_rng(seed)
    rows = set(g.choice(M, size=n - 2, replace=False).tolist()) | {0, M - 1}
    return np.array(sorted(rows))


def assert_close(Y, oracle_lib, X, W, bits, keep, rows=None, what=""):
    Xc, Wc = X.cpu(), W.cpu()
    Yo, _ = oracle_lib.linear(Xc, Wc, bits.cpu().numpy(), rows=rows)
    Wm = oracle_lib.apply_mask(Wc, keep.cpu().numpy().astype(np.uint8))
    S = oracle_lib.abs_scale(Xc, Wm, rows=rows)
    Yg = Y.float().cpu().numpy()
    if rows is not None:
        Yg = Yg[rows]
    assert np.isfinite(Yg).all(), f"{what}: non-finite output"
    err = np.abs(Yg - Yo)
    bad = err > TOL_ELEM * S
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} outside tolerance, "
                           f"worst err {err[bad].max()} at scale {S[bad][np.argmax(err[bad])]}")
    denom = np.linalg.norm(Yo)
    if denom > 0:
        fro = np.linalg.norm(Yg - Yo) / denom
        assert fro <= TOL_FRO, f"{what}: relative Frobenius error {fro}"
    else:
        assert np.all(Yg == 0)


def pack(hsg, p):
    return hsg.PackedLinear.pack(p.W, p.bits, p.flags.cpu(), p.R, p.C, bitorder=p.bitorder)


def check_pack(hsg, oracle_lib, p, lin):
    packed, (slab, meta, gemm) = lin.packed()
    keep = p.keep.cpu().numpy().astype(np.uint8)
    op, ot = oracle_lib.pack(p.W.cpu(), keep, p.flags.cpu().numpy().reshape(-1), p.R, p.C)
    assert np.array_equal(slab, ot.slab) and np.array_equal(meta, ot.meta) and np.array_equal(gemm, ot.gemm)
    assert packed.size == op.size
    diff = np.flatnonzero(packed != op)
    assert diff.size == 0, f"{diff.size} packed bytes differ, first at {diff[:8]}"


# ------------------------------------------------------------------ pack ---

@pytest.mark.parametrize("R,C", [(128, 128), (128, 64), (64, 128), (64, 64)])
@pytest.mark.parametrize("frac", [0.0, 0.5, 1.0])
@pytest.mark.parametrize("bitorder", [0, 1])
@pytest.mark.parametrize("N", [256, 384])
def test_pack_bit_exact(hsg, oracle_lib, R, C, frac, bitorder, N):
    K = 448 if C == 64 else 384
    p = synth.make_problem(N, K, 0, R=R, C=C, frac=frac, seed=7, device="cuda", bitorder=bitorder)
    lin = pack(hsg, p)
    check_pack(hsg, oracle_lib, p, lin)
    info = lin.info()
    assert info.tiles_sparse == int(p.flags.sum())
    assert info.pruned == int((~p.keep).sum())
    assert info.stray_zeros == 0
    Wm = lin.unpack()
    torch.cuda.synchronize()
    ref = oracle_lib.apply_mask(p.W.cpu(), p.keep.cpu().numpy().astype(np.uint8))
    assert np.array_equal(Wm.cpu().view(torch.int16).numpy().view(np.uint16), ref)
    lin.free()


def test_pack_rejects_bad_mask(hsg):
    p = synth.make_problem(256, 256, 0, frac=1.0, seed=1, device="cuda")
    keep = p.keep.clone()
    keep[5, 8:12] = True  # four kept in one group of a 2:4 tile
    bits = synth.pack_bits(keep)
    with pytest.raises(hsg.PatchError) as e:
        hsg.PackedLinear.pack(p.W, bits, p.flags.cpu())
    assert e.value.status == 4


def test_stray_zeros_in_dense_tiles(hsg, oracle_lib):
    p = synth.make_problem(256, 256, 32, frac=0.5, seed=2, device="cuda")
    keep = p.keep.clone()
    fl = p.flags.cpu().numpy()
    ti, tj = np.argwhere(fl == 0)[0]
    keep[ti * 128 + 3, tj * 128 + 10] = False
    keep[ti * 128 + 77, tj * 128 + 100] = False
    bits = synth.pack_bits(keep)
    lin = hsg.PackedLinear.pack(p.W, bits, p.flags.cpu())
    assert lin.info().stray_zeros == 2
    Y = lin(p.X, path=hsg.PATH_GEMM)
    torch.cuda.synchronize()
    assert_close(Y, oracle_lib, p.X, p.W, bits, keep, what="stray zeros")
    lin.free()


# --------------------------------------------------------------- product ---

SMALL = [(256, 384, 128, 128), (384, 448, 128, 64), (256, 512, 64, 128), (384, 320, 64, 64)]


SMALL_ODD = SMALL + [(640, 320, 128, 64), (128, 256, 128, 128)]  # odd strip counts


@pytest.mark.parametrize("N,K,R,C", SMALL_ODD)
@pytest.mark.parametrize("frac", [0.0, 0.6, 1.0])
@pytest.mark.parametrize("M", [1, 5, 16, 17, 128, 129, 300])
@pytest.mark.parametrize("kernel", ["single", "pair"])
def test_gemm_small(hsg, oracle_lib, N, K, R, C, frac, M, kernel):
    p = synth.make_problem(N, K, M, R=R, C=C, frac=frac, seed=M, device="cuda")
    lin = pack(hsg, p)
    path = hsg.PATH_GEMM_SINGLE if kernel == "single" else hsg.PATH_GEMM_PAIR
    Y = lin(p.X, path=path)
    torch.cuda.synchronize()
    lin.check()
    assert_close(Y, oracle_lib, p.X, p.W, p.bits, p.keep, what=f"{kernel} M={M}")
    lin.free()


@pytest.mark.parametrize("M", [256, 511, 700, 1024])
@pytest.mark.parametrize("frac", [0.3, 0.9])
def test_pair_tiles_several_blocks(hsg, oracle_lib, M, frac):
    """Several 256-token blocks and strip pairs per CTA pair, mixed kinds in a pair."""
    p = synth.make_problem(1152, 1024, M, R=128, C=128, frac=frac, seed=M, device="cuda")
    lin = pack(hsg, p)
    info = lin.info()
    assert info.dense_images == info.slabs_sparse - info.slabs_pair_sparse
    for path in (hsg.PATH_GEMM_PAIR, hsg.PATH_GEMM_SINGLE, hsg.PATH_GEMM):
        Y = lin(p.X, path=path)
        torch.cuda.synchronize()
        lin.check()
        assert_close(Y, oracle_lib, p.X, p.W, p.bits, p.keep, rows=sample_rows(M, 96, M),
                     what=f"pair blocks path {path}")
    lin.free()


@pytest.mark.parametrize("N,K,R,C", SMALL_ODD)
@pytest.mark.parametrize("frac", [0.0, 0.6, 1.0])
@pytest.mark.parametrize("M", [1, 2, 3, 4, 7, 8, 12, 16])
@pytest.mark.parametrize("kernel", ["tc", "simt"])
def test_gemv_small(hsg, oracle_lib, N, K, R, C, frac, M, kernel):
    p = synth.make_problem(N, K, M, R=R, C=C, frac=frac, seed=M + 100, device="cuda")
    lin = pack(hsg, p)
    Y = lin(p.X, path=hsg.PATH_GEMV if kernel == "tc" else hsg.PATH_GEMV_SIMT)
    torch.cuda.synchronize()
    lin.check()
    assert_close(Y, oracle_lib, p.X, p.W, p.bits, p.keep, what=f"gemv {kernel} M={M}")
    lin.free()


@pytest.mark.parametrize("N,K,R,C", SMALL_ODD)
@pytest.mark.parametrize("frac", [0.0, 0.6, 1.0])
@pytest.mark.parametrize("M", [17, 31, 33, 48, 63, 64])
def test_decode_wide_small(hsg, oracle_lib, N, K, R, C, frac, M):
    """The decode kernel's 64-token instance (16 < M <= 64): ragged M inside
    its one token tile, every tile shape and fraction."""
    p = synth.make_problem(N, K, M, R=R, C=C, frac=frac, seed=M + 300, device="cuda")
    lin = pack(hsg, p)
    Y = lin(p.X, path=hsg.PATH_GEMV)
    torch.cuda.synchronize()
    lin.check()
    assert_close(Y, oracle_lib, p.X, p.W, p.bits, p.keep, what=f"decode wide M={M}")
    lin.free()


def test_decode_repeat_and_interleave(hsg, oracle_lib):
    """The split-K decode re-arms its per-strip counters: repeated and
    interleaved calls on one handle give identical bits."""
    p = synth.make_problem(1152, 2048, 64, R=128, C=128, frac=0.7, seed=9, device="cuda")
    lin = pack(hsg, p)
    outs = []
    # both instances (16- and 64-token MMAs) share the per-strip counters
    for M in (16, 1, 64, 16, 5, 40, 16, 64):
        X = p.X[:M].contiguous()
        outs.append((M, lin(X, path=hsg.PATH_GEMV)))
    torch.cuda.synchronize()
    lin.check()
    assert torch.equal(outs[0][1], outs[3][1]) and torch.equal(outs[0][1], outs[6][1])
    assert torch.equal(outs[2][1], outs[7][1])
    for M, Y in outs:
        assert_close(Y, oracle_lib, p.X[:M].contiguous(), p.W, p.bits, p.keep, what=f"decode repeat M={M}")
    lin.free()


@pytest.mark.parametrize("N", [128, 384, 512, 640, 1152])
@pytest.mark.parametrize("M", [16, 100, 240, 241, 497, 1000])
@pytest.mark.parametrize("R,C,frac", [(128, 128, 0.9), (64, 64, 0.3), (128, 64, 1.0), (64, 128, 0.0)])
def test_wide_tiles(hsg, oracle_lib, N, M, R, C, frac):
    """Two strips per CTA of a pair: strip counts that leave one, two or three
    strips of the last quad as duplicates, token counts that end in a ragged
    tile (a narrower MMA) or fill tiles exactly."""
    p = synth.make_problem(N, 512, M, R=R, C=C, frac=frac, seed=3 * N + M, device="cuda", tag="wide")
    lin = pack(hsg, p)
    Y = lin(p.X, path=hsg.PATH_GEMM_WIDE)
    Y2 = lin(p.X, path=hsg.PATH_GEMM_WIDE)
    torch.cuda.synchronize()
    lin.check()
    assert torch.equal(Y, Y2)
    assert_close(Y, oracle_lib, p.X, p.W, p.bits, p.keep, rows=sample_rows(M, 96, N), what=f"wide N={N} M={M}")
    lin.free()


@pytest.mark.parametrize("K,C", [(64, 64), (128, 128), (192, 64)])
@pytest.mark.parametrize("frac", [0.0, 0.5, 1.0])
def test_wide_short_k(hsg, oracle_lib, K, C, frac):
    """One to three slabs per tile: many tiles pass through the slab ring and
    its per-slab barriers in one launch (both kinds of record mixed)."""
    p = synth.make_problem(1024, K, 2000, R=128, C=C, frac=frac, seed=K, device="cuda", tag="wides")
    lin = pack(hsg, p)
    Y = lin(p.X, path=hsg.PATH_GEMM_WIDE)
    torch.cuda.synchronize()
    lin.check()
    assert torch.equal(Y, lin(p.X, path=hsg.PATH_GEMM_PAIR))
    assert_close(Y, oracle_lib, p.X, p.W, p.bits, p.keep, rows=sample_rows(2000, 48, K), what=f"wide K={K}")
    lin.free()


def test_wide_long_k(hsg, oracle_lib):
    """Many slabs per tile (K = 4096) and several tiles per CTA pair."""
    p = synth.make_problem(1024, 4096, 2000, R=128, C=128, frac=0.7, seed=11, device="cuda", tag="widek")
    lin = pack(hsg, p)
    Y = lin(p.X, path=hsg.PATH_GEMM_WIDE)
    torch.cuda.synchronize()
    lin.check()
    assert_close(Y, oracle_lib, p.X, p.W, p.bits, p.keep, rows=sample_rows(2000, 48, 5), what="wide long K")
    lin.free()


@pytest.mark.parametrize("frac", [0.6, 1.0])
def test_wide_tables_beyond_shared_copy(hsg, oracle_lib, frac):
    """K = 16448 (257 slabs per strip): more records than the producers copy
    into shared memory, so the general instance reads its tables from global
    memory; the pure 2:4 instance computes them. A K % 128 == 64 tail too."""
    p = synth.make_problem(512, 16448, 300, R=128, C=64, frac=frac, seed=13, device="cuda", tag="widetab")
    lin = pack(hsg, p)
    Y = lin(p.X, path=hsg.PATH_GEMM_WIDE)
    torch.cuda.synchronize()
    lin.check()
    assert_close(Y, oracle_lib, p.X, p.W, p.bits, p.keep, rows=sample_rows(300, 24, 6), what=f"wide K=16448 f={frac}")
    lin.free()


def test_large_m_and_wide_n(hsg, oracle_lib):
    """Maximum-size cases on small weights: 100003 tokens (hundreds of token
    tiles, ragged last tile, Y beyond 2^26 elements) through every large-M
    kernel, and a 28672-row linear (224 strips) on the decode and automatic
    paths; sampled rows (first and last included) against the oracle."""
    p = synth.make_problem(512, 256, 100003, R=128, C=128, frac=0.7, seed=41, device="cuda", tag="bigM")
    lin = pack(hsg, p)
    rows = sample_rows(p.X.shape[0], 96, 41)
    for path in (hsg.PATH_GEMM_WIDE, hsg.PATH_GEMM_PAIR, hsg.PATH_GEMM_SINGLE, hsg.PATH_AUTO):
        Y = lin(p.X, path=path)
        torch.cuda.synchronize()
        lin.check()
        assert_close(Y, oracle_lib, p.X, p.W, p.bits, p.keep, rows=rows, what=f"M=100003 path {path}")
        del Y
    lin.free()
    q = synth.make_problem(28672, 256, 300, R=128, C=64, frac=0.5, seed=42, device="cuda", tag="bigN")
    lin = pack(hsg, q)
    for path, M in ((hsg.PATH_GEMV, 37), (hsg.PATH_GEMV, 3), (hsg.PATH_AUTO, 300)):
        X = q.X[:M].contiguous()
        Y = lin(X, path=path)
        torch.cuda.synchronize()
        lin.check()
        assert_close(Y, oracle_lib, X, q.W, q.bits, q.keep, what=f"N=28672 path {path} M={M}")
    lin.free()


def test_single_strip_single_slab(hsg, oracle_lib):
    for frac in (0.0, 1.0):
        p = synth.make_problem(128, 64, 9, R=128, C=64, frac=frac, seed=3, device="cuda")
        lin = pack(hsg, p)
        for path in (hsg.PATH_GEMM_SINGLE, hsg.PATH_GEMM_PAIR, hsg.PATH_GEMV, hsg.PATH_GEMV_SIMT):
            Y = lin(p.X, path=path)
            torch.cuda.synchronize()
            assert_close(Y, oracle_lib, p.X, p.W, p.bits, p.keep, what=f"single slab {path}")
        # the decode kernel's 64-token instance on the one slab
        X = synth.normal_bf16((57, 64), 1.0, "cuda", "single-slab", frac)
        Y = lin(X, path=hsg.PATH_GEMV)
        torch.cuda.synchronize()
        assert_close(Y, oracle_lib, X, p.W, p.bits, p.keep, what="single slab, 57 tokens")
        lin.free()


def test_zero_weights_and_checkerboard(hsg, oracle_lib):
    N, K = 256, 256
    W = torch.zeros(N, K, dtype=torch.bfloat16, device="cuda")
    fl = torch.from_numpy((np.indices((N // 64, K // 64)).sum(0) % 2).astype(np.uint8))
    keep = synth.top2_keep(W, fl, 64, 64)  # ties -> lowest two positions kept
    bits = synth.pack_bits(keep)
    X = synth.normal_bf16((40, K), 1.0, "cuda", "zero", "X")
    lin = hsg.PackedLinear.pack(W, bits, fl, 64, 64)
    for path, M in ((hsg.PATH_GEMM_SINGLE, 40), (hsg.PATH_GEMM_PAIR, 40), (hsg.PATH_GEMV, 16),
                    (hsg.PATH_GEMV, 40), (hsg.PATH_GEMV_SIMT, 16)):
        Y = lin(X[:M].contiguous(), path=path)
        torch.cuda.synchronize()
        assert torch.count_nonzero(Y.float()) == 0
    lin.free()
    # checkerboard with real weights
    p = synth.make_problem(N, K, 33, R=64, C=64, seed=4, device="cuda")
    keep = synth.top2_keep(p.W, fl, 64, 64)
    bits = synth.pack_bits(keep)
    lin = hsg.PackedLinear.pack(p.W, bits, fl, 64, 64)
    assert lin.info().slabs_sparse == 0
    for path in (hsg.PATH_GEMM_SINGLE, hsg.PATH_GEMM_PAIR, hsg.PATH_GEMV):
        Y = lin(p.X, path=path)
        torch.cuda.synchronize()
        assert_close(Y, oracle_lib, p.X, p.W, bits, keep, what="checkerboard")
    lin.free()


def test_one_sparse_tile(hsg, oracle_lib):
    p = synth.make_problem(512, 512, 50, R=128, C=128, n_sparse=1, seed=5, device="cuda")
    lin = pack(hsg, p)
    for path, M in ((hsg.PATH_GEMM_SINGLE, 50), (hsg.PATH_GEMM_PAIR, 50), (hsg.PATH_GEMV, 16),
                    (hsg.PATH_GEMV, 50), (hsg.PATH_GEMV_SIMT, 16)):
        X = p.X[:M].contiguous()
        Y = lin(X, path=path)
        torch.cuda.synchronize()
        assert_close(Y, oracle_lib, X, p.W, p.bits, p.keep, what=f"one sparse tile {path}")
    lin.free()


def test_empty_and_misaligned(hsg):
    p = synth.make_problem(256, 256, 8, seed=6, device="cuda")
    lin = pack(hsg, p)
    Y = torch.full((0, 256), 7.0, dtype=torch.bfloat16, device="cuda")
    lin(p.X[:0], out=Y)  # M = 0: nothing to do
    buf = torch.zeros(8 * 256 + 8, dtype=torch.bfloat16, device="cuda")
    Xmis = buf[1:1 + 8 * 256].view(8, 256)
    with pytest.raises(hsg.PatchError) as e:
        lin(Xmis)
    assert e.value.status == 3
    with pytest.raises(hsg.PatchError) as e:  # the decode kernel takes M <= 64
        lin(torch.zeros(65, 256, dtype=torch.bfloat16, device="cuda"), path=hsg.PATH_GEMV)
    assert e.value.status == 2
    with pytest.raises(hsg.PatchError) as e:  # the CUDA-core one M <= 16
        lin(torch.zeros(17, 256, dtype=torch.bfloat16, device="cuda"), path=hsg.PATH_GEMV_SIMT)
    assert e.value.status == 2
    lin.free()


def test_decode_concurrent_streams(hsg, oracle_lib):
    """Decode calls on one handle and on one group from two streams, with no
    synchronisation between the streams: each stream has its own split-K
    workspace, so both streams' results equal the sequential ones bit for bit
    (and the oracle)."""
    p = synth.make_problem(1152, 4096, 64, R=128, C=128, frac=0.7, seed=19, device="cuda")
    q = synth.make_problem(640, 4096, 16, R=128, C=128, frac=0.5, seed=20, device="cuda")
    lp, lq = pack(hsg, p), pack(hsg, q)
    g = hsg.LinearGroup([lp, lq])
    Xa, Xb, Xw = p.X[:16].contiguous(), p.X[:3].contiguous(), p.X[:50].contiguous()
    ref_a, ref_b = lp(Xa, path=hsg.PATH_GEMV), lp(Xb, path=hsg.PATH_GEMV)
    ref_w = lp(Xw, path=hsg.PATH_GEMV)
    gref = g([Xa, q.X[:16].contiguous()], path=hsg.PATH_GEMV)
    torch.cuda.synchronize()
    sa, sb = torch.cuda.Stream(), torch.cuda.Stream()
    outs_a, outs_b, outs_w, gouts = [], [], [], []
    for _ in range(20):
        outs_a.append(lp(Xa, path=hsg.PATH_GEMV, stream=sa))
        outs_w.append(lp(Xw, path=hsg.PATH_GEMV, stream=sa))
        outs_b.append(lp(Xb, path=hsg.PATH_GEMV, stream=sb))
        gouts.append(g([Xa, q.X[:16].contiguous()], path=hsg.PATH_GEMV, stream=sb))
    torch.cuda.synchronize()
    lp.check()
    for Ya, Yb, Yw, Yg in zip(outs_a, outs_b, outs_w, gouts):
        assert torch.equal(Ya, ref_a) and torch.equal(Yb, ref_b) and torch.equal(Yw, ref_w)
        assert torch.equal(Yg[0], gref[0]) and torch.equal(Yg[1], gref[1])
    assert_close(outs_w[-1], oracle_lib, Xw, p.W, p.bits, p.keep, what="decode stream a, 64-token instance")
    assert_close(outs_a[-1], oracle_lib, Xa, p.W, p.bits, p.keep, what="decode stream a")
    assert_close(outs_b[-1], oracle_lib, Xb, p.W, p.bits, p.keep, what="decode stream b")
    g.free()
    lp.free()
    lq.free()


def test_first_call_schedule_used_from_another_stream(hsg, oracle_lib):
    """The first call for an M uploads its schedule asynchronously; a call on
    another stream right after it (no host synchronisation) waits for the
    upload on the device and gives the same bits."""
    p = synth.make_problem(1024, 2048, 777, R=128, C=128, frac=0.9, seed=23, device="cuda")
    lin = pack(hsg, p)
    sa, sb = torch.cuda.Stream(), torch.cuda.Stream()
    Ya = lin(p.X, stream=sa)
    Yb = lin(p.X, stream=sb)
    torch.cuda.synchronize()
    assert torch.equal(Ya, Yb)
    rows = sample_rows(777)
    assert_close(Yb, oracle_lib, p.X, p.W, p.bits, p.keep, rows=rows, what="schedule from another stream")
    lin.free()


@pytest.mark.parametrize("M", [5, 40, 100, 300, 1000, 2048])
def test_group_host_matches_device(hsg, M):
    """patch_group_linear_host (token chunks whose copies overlap the product)
    gives the device call's bits; members sharing a host input (q, k, v) and
    two calls in a row without a host synchronisation between them."""
    shapes = [(512, 1024), (256, 1024), (384, 768)]
    probs = [synth.make_problem(N, K, M, R=128, C=128, frac=0.7, seed=40 + i, device="cuda", tag="gh")
             for i, (N, K) in enumerate(shapes)]
    lins = [pack(hsg, p) for p in probs]
    g = hsg.LinearGroup(lins)
    X1 = probs[0].X
    Xs_dev = [X1, X1, probs[2].X]
    ref = g(Xs_dev)
    torch.cuda.synchronize()
    xa = X1.cpu().pin_memory()
    Xh = [xa, xa, probs[2].X.cpu().pin_memory()]
    out1 = g.host(Xh, sync=False)
    Xh2 = [x.clone().pin_memory() for x in Xh]
    out2 = g.host(Xh2, sync=False)
    torch.cuda.synchronize()
    for o1, o2, r in zip(out1, out2, ref):
        assert torch.equal(o1, r.cpu()) and torch.equal(o2, r.cpu())
    # pageable host memory works too (copies block the host)
    out3 = g.host([x.clone() for x in Xh], outs=[torch.empty_like(r, device="cpu") for r in ref])
    for o, r in zip(out3, ref):
        assert torch.equal(o, r.cpu())
    g.free()
    for l in lins:
        l.free()


def test_cuda_graph_capture_and_replay(hsg):
    """After one call with the same M has completed, patch_linear and
    patch_group_linear calls (tensor-core GEMM and decode) can be captured in
    a CUDA graph; replays give the eager bits."""
    p = synth.make_problem(1024, 2048, 600, R=128, C=128, frac=0.7, seed=29, device="cuda")
    q = synth.make_problem(512, 2048, 600, R=128, C=128, frac=0.9, seed=30, device="cuda")
    lp, lq = pack(hsg, p), pack(hsg, q)
    g = hsg.LinearGroup([lp, lq])
    X16 = p.X[:16].contiguous()
    X48 = [p.X[:48].contiguous(), q.X[:48].contiguous()]
    Y1 = torch.empty((600, 1024), dtype=torch.bfloat16, device="cuda")
    Y2 = torch.empty((16, 1024), dtype=torch.bfloat16, device="cuda")
    G = [torch.empty((600, 1024), dtype=torch.bfloat16, device="cuda"),
         torch.empty((600, 512), dtype=torch.bfloat16, device="cuda")]
    G48 = [torch.empty((48, 1024), dtype=torch.bfloat16, device="cuda"),
           torch.empty((48, 512), dtype=torch.bfloat16, device="cuda")]
    eager1, eager2 = lp(p.X), lp(X16)
    eg = g([p.X, q.X])
    eg48 = g(X48, path=hsg.PATH_GEMV)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        lp(p.X, out=Y1)
        lp(X16, out=Y2)
        g([p.X, q.X], G)
        g(X48, G48, path=hsg.PATH_GEMV)
    for _ in range(3):
        for t in (Y1, Y2, *G, *G48):
            t.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(Y1, eager1) and torch.equal(Y2, eager2)
        assert torch.equal(G[0], eg[0]) and torch.equal(G[1], eg[1])
        assert torch.equal(G48[0], eg48[0]) and torch.equal(G48[1], eg48[1])
    lp.check()
    del graph
    g.free()
    lp.free()
    lq.free()


def test_deterministic_and_host_path(hsg):
    p = synth.make_problem(512, 1024, 300, R=128, C=64, frac=0.7, seed=8, device="cuda")
    lin = pack(hsg, p)
    for path in (hsg.PATH_GEMM_SINGLE, hsg.PATH_GEMM_PAIR, hsg.PATH_GEMM):
        Ya = lin(p.X, path=path)
        Yb = lin(p.X, path=path)
        torch.cuda.synchronize()
        assert torch.equal(Ya, Yb)
    Y1 = lin(p.X)
    torch.cuda.synchronize()
    Yh = lin.host(p.X.cpu().pin_memory())
    assert torch.equal(Yh, Y1.cpu())
    Xs = p.X[:5].contiguous()
    Yh5 = lin.host(Xs.cpu())
    assert torch.equal(Yh5, lin(Xs).cpu())
    lin.free()


def test_gemm_and_gemv_agree_with_oracle_on_config_1(hsg, oracle_lib):
    """512x512 layer, M = 16, a 4x4 grid of 128x128 tiles with 8 seeded 2:4 tiles."""
    p = synth.make_problem(512, 512, 16, R=128, C=128, n_sparse=8, seed=0, device="cuda")
    lin = pack(hsg, p)
    check_pack(hsg, oracle_lib, p, lin)
    assert abs(lin.info().sparsity - 0.25) < 1e-12
    for path in (hsg.PATH_GEMM_SINGLE, hsg.PATH_GEMM_PAIR, hsg.PATH_GEMV, hsg.PATH_GEMV_SIMT, hsg.PATH_AUTO):
        Y = lin(p.X, path=path)
        torch.cuda.synchronize()
        assert_close(Y, oracle_lib, p.X, p.W, p.bits, p.keep, what=f"config1 {path}")
    lin.free()


# ------------------------------------------------------ full-size workloads ---

def _layer(hsg, oracle_lib, shapes, M, fracs, R=128, C=128, seed=0, tag="cfg", paths=None,
           check_bytes=False, rows_n=128):
    X_by_k = {}
    for lin_shape, f in zip(shapes, fracs):
        N, K = lin_shape.N, lin_shape.K
        if K not in X_by_k:
            X_by_k[K] = synth.normal_bf16((M, K), 1.0, "cuda", tag, "X", seed, M, K)
        X = X_by_k[K]
        T = (N // R) * (K // C)
        p = synth.make_problem(N, K, 0, R=R, C=C, n_sparse=int(round(f * T)), seed=seed,
                               device="cuda", tag=f"{tag}-{lin_shape.name}")
        lin = pack(hsg, p)
        if check_bytes:
            check_pack(hsg, oracle_lib, p, lin)
        rows = sample_rows(M, rows_n, seed)
        for path in (paths or [hsg.PATH_AUTO]):
            Y = lin(X, path=path)
            torch.cuda.synchronize()
            lin.check()
            assert_close(Y, oracle_lib, X, p.W, p.bits, p.keep, rows=None if M <= rows_n else rows,
                         what=f"{tag} {lin_shape.name} path {path}")
        lin.free()
        del p


def test_config2_llama32_1b_m4096(hsg, oracle_lib):
    shapes = synth.llama32_1b()
    T = [(l.N // 128) * (l.K // 128) for l in shapes]
    cnt = synth.split_fraction(T, 0.9, 0.8, 1.0, "cfg2")
    _layer(hsg, oracle_lib, shapes, 4096, [c / t for c, t in zip(cnt, T)], tag="cfg2", check_bytes=True)


@pytest.mark.parametrize("model,M", [("llama32_1b", 4096), ("llama2_7b", 2048)])
def test_grouped_layer_as_benchmarked(hsg, oracle_lib, model, M):
    """The launch the bench times: one layer's seven linears in one grouped
    launch on the two-strips-per-CTA kernel, sampled rows against the oracle."""
    shapes = getattr(synth, model)()
    T = [(l.N // 128) * (l.K // 128) for l in shapes]
    cnt = synth.split_fraction(T, 0.9, 0.8, 1.0, f"grp-{model}")
    X_by_k = {K: synth.normal_bf16((M, K), 1.0, "cuda", "grp", "X", 0, M, K) for K in sorted({l.K for l in shapes})}
    probs = [synth.make_problem(l.N, l.K, 0, n_sparse=c, seed=0, device="cuda", tag=f"grp-{model}-{l.name}")
             for l, c in zip(shapes, cnt)]
    lins = [pack(hsg, p) for p in probs]
    g = hsg.LinearGroup(lins)
    assert g.path(M) == hsg.PATH_GEMM_WIDE
    Ys = g([X_by_k[l.K] for l in shapes])
    torch.cuda.synchronize()
    lins[0].check()
    rows = sample_rows(M, 64, 1)
    for l, p, Y in zip(shapes, probs, Ys):
        assert_close(Y, oracle_lib, X_by_k[l.K], p.W, p.bits, p.keep, rows=rows, what=f"{model} grouped {l.name}")
    g.free()
    for lin in lins:
        lin.free()


@pytest.mark.parametrize("model,M,members", [("llama2_7b", 2048, None), ("llama2_13b", 8192, ["q", "up", "down"])])
def test_pure_24_instance(hsg, oracle_lib, model, M, members):
    """Pure 2:4 weights (every tile 2:4, the MaskLLM end of the range) run the
    wide kernel's pure instance, which computes each record's place instead
    of reading the tables: a Llama-2-7B layer at M = 2048 and Llama-2-13B
    linears at M = 8192. AUTO picks it, an explicit request gives the same
    bits, and sampled rows match the oracle."""
    shapes = [l for l in getattr(synth, model)() if members is None or l.name in members]
    X_by_k = {K: synth.normal_bf16((M, K), 1.0, "cuda", "pure", "X", 0, M, K) for K in sorted({l.K for l in shapes})}
    probs = [synth.make_problem(l.N, l.K, 0, frac=1.0, seed=0, device="cuda", tag=f"pure-{model}-{l.name}")
             for l in shapes]
    lins = [pack(hsg, p) for p in probs]
    for lin in lins:
        info = lin.info()
        assert info.slabs_pair_sparse == info.slabs_total and info.dense_images == 0
        assert abs(info.sparsity - 0.5) < 1e-12
    g = hsg.LinearGroup(lins)
    assert g.path(M) == hsg.PATH_GEMM_WIDE_24
    xs = [X_by_k[l.K] for l in shapes]
    Ys = g(xs)
    Ys2 = g(xs, path=hsg.PATH_GEMM_WIDE_24)
    torch.cuda.synchronize()
    lins[0].check()
    assert all(torch.equal(a, b) for a, b in zip(Ys, Ys2))
    rows = sample_rows(M, 48, 2)
    for l, p, Y in zip(shapes, probs, Ys):
        assert_close(Y, oracle_lib, X_by_k[l.K], p.W, p.bits, p.keep, rows=rows, what=f"{model} pure 2:4 {l.name}")
    g.free()
    for lin in lins:
        lin.free()


@pytest.mark.parametrize("M", [1, 4, 16, 32, 64])
def test_config3_llama2_7b_decode(hsg, oracle_lib, M):
    shapes = synth.llama2_7b()
    paths = [hsg.PATH_GEMV, hsg.PATH_GEMM] + ([hsg.PATH_GEMV_SIMT] if M <= 16 else [])
    _layer(hsg, oracle_lib, shapes, M, [0.7] * 7, tag="cfg3", paths=paths, check_bytes=(M == 1))


@pytest.mark.parametrize("frac", [0.0, 0.5, 0.7, 0.9, 1.0])
def test_config4_llama2_7b_prefill_sweep(hsg, oracle_lib, frac):
    shapes = synth.llama2_7b()
    _layer(hsg, oracle_lib, shapes, 2048, [frac] * 7, tag=f"cfg4-{frac}", rows_n=64)


@pytest.mark.parametrize("R,C", [(128, 128), (128, 64), (64, 128), (64, 64)])
def test_config5_llama2_13b_tiles(hsg, oracle_lib, R, C):
    shapes = [l for l in synth.llama2_13b() if l.name in ("q", "gate", "down")]
    _layer(hsg, oracle_lib, shapes, 8192, [0.9] * 3, R=R, C=C, tag=f"cfg5-{R}x{C}", rows_n=64,
           check_bytes=(R == 64 and C == 64))


# --------------------------------------------------------------- groups ---

@pytest.mark.parametrize("path_name,M", [("GEMM_PAIR", 300), ("GEMM_SINGLE", 130), ("GEMV", 16), ("GEMV", 3),
                                         ("GEMV_SIMT", 5), ("AUTO", 520), ("AUTO", 1), ("GEMM_WIDE", 300),
                                         ("GEMM_WIDE", 17), ("GEMV", 40), ("GEMV", 64)])
def test_group_matches_members(hsg, oracle_lib, path_name, M):
    """One launch over several linears (shared and separate inputs, mixed tile
    shapes and 2:4 fractions) equals the members run one by one, bit for bit,
    and each member is within tolerance of the oracle."""
    specs = [(384, 256, 128, 128, 0.9, "a"), (128, 256, 128, 64, 0.5, "a"), (640, 384, 64, 64, 0.7, "b"),
             (256, 448, 128, 64, 0.0, "c")]
    Xs = {"a": synth.normal_bf16((M, 256), 1.0, "cuda", "gx", "a", M),
          "b": synth.normal_bf16((M, 384), 1.0, "cuda", "gx", "b", M),
          "c": synth.normal_bf16((M, 448), 1.0, "cuda", "gx", "c", M)}
    probs, lins, xs = [], [], []
    for i, (N, K, R, C, f, xk) in enumerate(specs):
        p = synth.make_problem(N, K, 0, R=R, C=C, frac=f, seed=i, device="cuda", tag=f"grp{i}")
        probs.append(p)
        lins.append(pack(hsg, p))
        xs.append(Xs[xk])
    path = getattr(hsg, "PATH_" + path_name)
    group = hsg.LinearGroup(lins)
    Yg = group(xs, path=path)
    Yi = [lin(x, path=path) for lin, x in zip(lins, xs)]
    torch.cuda.synchronize()
    lins[0].check()
    # the decode kernel may split K differently inside a group (different
    # summation order); every other kernel gives the same bits
    decode = path == hsg.PATH_GEMV or (path == hsg.PATH_AUTO and M <= 64)
    for i, (p, x) in enumerate(zip(probs, xs)):
        if not decode:
            assert torch.equal(Yg[i], Yi[i]), f"member {i} differs from its own launch"
        assert_close(Yg[i], oracle_lib, x, p.W, p.bits, p.keep, rows=sample_rows(M, 64, i),
                     what=f"group {path_name} member {i}")
    # a second call reuses the cached schedule
    Yg2 = group(xs, path=path)
    torch.cuda.synchronize()
    assert all(torch.equal(a, b) for a, b in zip(Yg, Yg2))
    group.free()
    for lin in lins:
        lin.free()


def test_group_path_choice(hsg):
    """AUTO resolves by M and by how many two-strip tiles the launch has."""
    small = pack(hsg, synth.make_problem(512, 256, 0, seed=1, device="cuda", tag="gp1"))
    big = pack(hsg, synth.make_problem(8192, 256, 0, seed=2, device="cuda", tag="gp2"))
    gs, gb = hsg.LinearGroup([small]), hsg.LinearGroup([big])
    assert gs.path(1) == hsg.PATH_GEMV and gs.path(16) == hsg.PATH_GEMV
    assert gs.path(17) == hsg.PATH_GEMV and gs.path(64) == hsg.PATH_GEMV
    assert gs.path(65) == hsg.PATH_GEMM_SINGLE and gs.path(255) == hsg.PATH_GEMM_SINGLE
    assert gs.path(256) == hsg.PATH_GEMM_PAIR          # one strip quad: too few tiles
    assert gb.path(4096) == hsg.PATH_GEMM_WIDE         # 16 quads x 18 token blocks
    assert gb.path(4096, hsg.PATH_GEMM_PAIR) == hsg.PATH_GEMM_PAIR
    assert gs.path(4, hsg.PATH_GEMV_SIMT) == hsg.PATH_GEMV_SIMT
    pure = pack(hsg, synth.make_problem(8192, 256, 0, frac=1.0, seed=3, device="cuda", tag="gp3"))
    gp = hsg.LinearGroup([pure])
    assert gp.path(4096) == hsg.PATH_GEMM_WIDE_24      # every slab 2:4: the pure instance
    assert gp.path(4096, hsg.PATH_GEMM_WIDE) == hsg.PATH_GEMM_WIDE_24
    assert gp.path(300, hsg.PATH_GEMM_PAIR) == hsg.PATH_GEMM_PAIR
    with pytest.raises(hsg.PatchError):
        gb([torch.empty((300, 256), dtype=torch.bfloat16, device="cuda")], path=hsg.PATH_GEMM_WIDE_24)
    for g in (gs, gb, gp):
        g.free()
    pure.free()
    small.free()
    big.free()


def test_device_wait_gives_up_and_context_survives(hsg, oracle_lib):
    """The bounded wait every kernel uses: a barrier nothing completes makes
    the kernel record a timeout and return (about 1 s); the error reaches the
    host as PATCH_ERR_TIMEOUT and the next product is still correct."""
    lib = hsg.library()
    assert lib.patch_selftest_wait(None) == 6          # PATCH_ERR_TIMEOUT
    assert b"gave up" in lib.patch_last_error()
    p = synth.make_problem(512, 512, 40, frac=0.5, seed=9, device="cuda", tag="after-timeout")
    lin = pack(hsg, p)
    Y = lin(p.X)
    torch.cuda.synchronize()
    lin.check()
    assert_close(Y, oracle_lib, p.X, p.W, p.bits, p.keep, what="after a device timeout")
    lin.free()


def test_group_argument_errors(hsg):
    import ctypes
    lib = hsg.library()
    g = ctypes.c_void_p()
    assert lib.patch_group_create(None, 1, ctypes.byref(g)) == 1
    p = synth.make_problem(128, 64, 0, R=128, C=64, seed=0, device="cuda", tag="ge")
    lin = pack(hsg, p)
    arr = (ctypes.c_void_p * 9)(*([lin.handle] * 9))
    assert lib.patch_group_create(arr, 9, ctypes.byref(g)) == 1
    assert lib.patch_group_create(arr, 0, ctypes.byref(g)) == 1
    assert lib.patch_group_linear(None, None, 4, None, 0, None) == 1
    lin.free()


# ------------------------------------------------ output-feature split ---

def test_row_sharded_single_rank_is_the_whole_linear(hsg):
    """One rank: the split is the whole weight, and the product is bit-equal
    to the unsplit linear's."""
    from hybrid_sparse_gemm_b200 import dist
    p = synth.make_problem(1280, 512, 300, R=64, C=128, frac=0.7, seed=21, device="cuda", tag="tp1")
    whole = pack(hsg, p)
    tp = dist.RowShardedLinear(p.W, p.bits, p.flags, p.R, p.C, rank=0, world=1)
    assert tp.bounds == [0, 1280]
    for M in (300, 5):
        X = p.X[:M].contiguous()
        assert torch.equal(tp(X), whole(X))
    torch.cuda.synchronize()
    tp.free()
    whole.free()


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("M", [300, 5])
def test_row_shards_assemble_the_product(hsg, oracle_lib, world, M):
    """Every rank's shard packed and run on this GPU in turn; its columns put
    side by side give the whole product within the parity bar."""
    from hybrid_sparse_gemm_b200 import dist
    p = synth.make_problem(1536, 512, M, R=128, C=128, frac=0.6, seed=22, device="cuda", tag=f"tp{world}")
    Y = torch.empty((M, 1536), dtype=torch.bfloat16, device="cuda")
    shards = [dist.RowShardedLinear(p.W, p.bits, p.flags, p.R, p.C, rank=r, world=world) for r in range(world)]
    for r, tp in enumerate(shards):
        n0, n1 = tp.bounds[r], tp.bounds[r + 1]
        assert n1 > n0
        Y[:, n0:n1] = tp.lin(p.X)
    torch.cuda.synchronize()
    assert_close(Y, oracle_lib, p.X, p.W, p.bits, p.keep, what=f"{world} shards, M={M}")
    for tp in shards:
        tp.free()
