"""Multi-rank host logic on CPU: gloo ranks in separate processes.

By tokens (data parallel) there is no collective on the data path, so what
needs checking across ranks is the timing reduction (the job takes as long as
its slowest rank), the whole-job rate, and that every rank draws its own
tokens while sharing the same weights.

By output features, each rank packs its cost-balanced block of W's rows and
one all-gather assembles Y. Here each rank's block product comes from the
oracle (the CUDA product needs a GPU); the assembled Y must equal the
oracle's product of the whole weight bit for bit, since every element of Y
depends only on its own row of W.
"""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    from hybrid_sparse_gemm_b200 import dist
    active = dist.init("gloo", timeout_s=30)
    assert active
    dist.barrier(active)
    ms = dist.max_over_ranks(1.5 + 2.0 * rank, active)
    # per-rank tokens, shared weights (the bench's seeding)
    x = synth.normal_bf16((4, 8), 1.0, "cpu", "X", 0, rank, 4, "q")
    w = synth.normal_bf16((8, 8), 0.02, "cpu", "W", 0, 8, 8, "q")
    xs = [torch.empty_like(x.float()) for _ in range(world)]
    ws = [torch.empty_like(w.float()) for _ in range(world)]
    torch.distributed.all_gather(xs, x.float())
    torch.distributed.all_gather(ws, w.float())
    out.put((rank, ms, all(torch.equal(ws[0], t) for t in ws), not torch.equal(xs[0], xs[1])))
    dist.shutdown(active)


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, same_w, diff_x in res:
        assert ms == 3.5          # the slowest rank's duration on every rank
        assert same_w and diff_x


def _nsplit_worker(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    from hybrid_sparse_gemm_b200 import dist
    active = dist.init("gloo", timeout_s=30)
    try:
        out.put((rank, _nsplit_cases(rank, world, active)))
    except Exception as e:  # report instead of leaving the parent waiting
        out.put((rank, repr(e)))
    dist.shutdown(active)


def _nsplit_cases(rank, world, active):
    import numpy as np
    import oracle
    import hybrid_sparse_gemm_b200 as hsg
    from hybrid_sparse_gemm_b200 import dist
    results = []
    for N, K, M, R, C, frac in ((1280, 256, 5, 64, 128, 0.6), (1536, 128, 3, 128, 64, 0.9), (384, 128, 2, 128, 128, 0.5)):
        p = synth.make_problem(N, K, M, R=R, C=C, frac=frac, seed=11, tag=f"ns{N}")
        bounds = hsg.patch_partition_rows(N, K, p.flags.numpy(), world, R, C)
        W, bits, _ = dist.shard_rows(p.W, p.bits, p.flags, R, bounds, rank)
        send, y_local = dist.local_buffer(M, bounds, rank, "cpu")
        if W.shape[0]:
            _, yb = oracle.linear(p.X, W, bits.numpy())
            y_local.copy_(torch.from_numpy(np.ascontiguousarray(yb).view(np.int16)).view(torch.bfloat16))
        Y = dist.gather_columns(send, M, bounds, active=active)
        _, full = oracle.linear(p.X, p.W, p.bits.numpy())
        results.append((bounds, torch.equal(Y.view(torch.int16), torch.from_numpy(np.ascontiguousarray(full).view(np.int16)))))
    return results


@pytest.mark.parametrize("world", [2, 3])
def test_output_feature_split_gloo(world, oracle_lib):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_nsplit_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(world):
        assert not isinstance(res[r], str), f"rank {r}: {res[r]}"
    for r in range(world):
        for (bounds, equal), (bounds0, _) in zip(res[r], res[0]):
            assert bounds == bounds0     # every rank computes the same split
            assert equal, f"rank {r}: assembled Y differs from the whole-weight oracle product ({bounds})"


def test_job_rate_and_single_rank():
    import sys
    sys.path.insert(0, ROOT)
    from hybrid_sparse_gemm_b200 import dist
    assert dist.job_rate(1e12, 4, 1000.0) == 4e12
    with pytest.raises(ValueError):
        dist.job_rate(1.0, 1, 0.0)
    assert dist.max_over_ranks(2.25, False) == 2.25
    assert dist.init("gloo") is False if os.environ.get("WORLD_SIZE", "1") == "1" else True
