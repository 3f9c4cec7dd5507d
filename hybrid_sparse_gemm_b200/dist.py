"""Process-group plumbing for multi-rank runs (one process per GPU).

Two ways to spread the hybrid linear over ranks:
  - by tokens (data parallel): every rank multiplies its own rows of X by a
    replicated packed weight. No exchange inside the layer; the only
    cross-rank steps are timing ones (a barrier before the timed region and
    the maximum of the per-rank durations after it).
  - by output features (tensor parallel, `RowShardedLinear`): each rank packs
    a contiguous block of W's rows, chosen by `patch_partition_rows` so that
    every rank has about the same tensor-core work, computes its columns of
    Y, and one all-gather assembles Y on every rank.
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as td


def env_ranks() -> tuple[int, int, int]:
    """(rank, local_rank, world_size) from the launcher's environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def init(backend: str, timeout_s: float = 120.0) -> bool:
    """Join the process group when the launcher started more than one rank.
    Returns True when a group is active."""
    _, _, world = env_ranks()
    if world <= 1:
        return False
    td.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
    return True


def barrier(active: bool) -> None:
    if active:
        td.barrier()


def max_over_ranks(value: float, active: bool, device="cpu") -> float:
    """Largest `value` over all ranks (the job is as slow as its slowest rank)."""
    if not active:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    td.all_reduce(t, op=td.ReduceOp.MAX)
    return float(t.item())


def job_rate(work_per_rank: float, world: int, ms_max: float) -> float:
    """Whole-job throughput: the work every rank did, over the slowest rank's time."""
    if ms_max <= 0:
        raise ValueError("duration must be positive")
    return world * work_per_rank / (ms_max / 1e3)


def shutdown(active: bool) -> None:
    if active:
        td.destroy_process_group()


# ------------------------------------------------ output-feature split ---

def shard_rows(W, mask_bits, tile_flags, tile_rows: int, bounds, rank: int):
    """Rows [bounds[rank], bounds[rank+1]) of W with their mask bits (row-major
    bit-packed, so a contiguous byte range) and their rows of tile flags: a
    valid patch_pack input. Views, no copies."""
    N, K = W.shape
    n0, n1 = int(bounds[rank]), int(bounds[rank + 1])
    if not (0 <= n0 <= n1 <= N) or n0 % tile_rows or n1 % tile_rows or (n0 * K) % 8:
        raise ValueError(f"bounds [{n0}, {n1}) do not cut whole tile rows of a {N}x{K} weight")
    flags = torch.as_tensor(tile_flags, dtype=torch.uint8).reshape(N // tile_rows, -1)
    return W[n0:n1], mask_bits.reshape(-1)[n0 * K // 8:n1 * K // 8], flags[n0 // tile_rows:n1 // tile_rows]


def local_buffer(M: int, bounds, rank: int, device, dtype=torch.bfloat16):
    """The send buffer of `gather_columns`, padded to the widest shard, and the
    M x n_rank row-major view of it that this rank's product is written into
    (so the exchange needs no extra copy on the sending side)."""
    world = len(bounds) - 1
    wmax = max(int(bounds[r + 1]) - int(bounds[r]) for r in range(world))
    n = int(bounds[rank + 1]) - int(bounds[rank])
    send = torch.empty(max(M * wmax, 1), dtype=dtype, device=device)
    return send, send[:M * n].view(M, n)


def gather_columns(send, M: int, bounds, out=None, active: bool = True, group=None):
    """The exchange step of the output-feature split. Rank r's `send` holds
    Y[:, bounds[r]:bounds[r+1]] as an M x n_r row-major block at its start;
    returns the whole M x N Y on every rank: one all-gather of the padded
    blocks, then each block copied into its columns."""
    world = len(bounds) - 1
    N = int(bounds[-1])
    widths = [int(bounds[r + 1]) - int(bounds[r]) for r in range(world)]
    if out is None:
        out = torch.empty((M, N), dtype=send.dtype, device=send.device)
    if world == 1:
        parts = [send]
    elif not active:
        raise ValueError("a split over several ranks needs an active process group")
    elif send.is_cuda:
        recv = torch.empty((world, send.numel()), dtype=send.dtype, device=send.device)
        td.all_gather_into_tensor(recv, send, group=group)
        parts = list(recv.unbind(0))
    else:
        # host tensors (gloo, which has no bf16): exchange the raw bytes
        wire = send.view(torch.uint8)
        parts = [torch.empty_like(wire) for _ in range(world)]
        td.all_gather(parts, wire, group=group)
        parts = [t.view(send.dtype) for t in parts]
    for r in range(world):
        if widths[r] and M:
            out[:, int(bounds[r]):int(bounds[r + 1])].copy_(parts[r][:M * widths[r]].view(M, widths[r]))
    return out


class RowShardedLinear:
    """One hybrid linear split by output features over the ranks of a process
    group. Every rank passes the whole W (or at least its rows), mask bits and
    tile flags; it packs only its own shard. Calling it with this rank's X
    (the same tokens on every rank) returns the whole Y on every rank."""

    def __init__(self, W, mask_bits, tile_flags, tile_rows: int = 128, tile_cols: int = 128, rank: int = 0,
                 world: int = 1, align_rows: int = 256, active: bool = False, group=None):
        from . import PackedLinear, patch_partition_rows
        N, K = W.shape
        self.N, self.K, self.rank, self.world = N, K, rank, world
        self.active, self.group = active, group
        self.bounds = patch_partition_rows(N, K, torch.as_tensor(tile_flags).cpu().numpy(), world, tile_rows,
                                           tile_cols, align_rows)
        Ws, bits, flags = shard_rows(W, mask_bits, tile_flags, tile_rows, self.bounds, rank)
        self.lin = (PackedLinear.pack(Ws.contiguous(), bits.contiguous(), flags.cpu(), tile_rows, tile_cols)
                    if Ws.shape[0] else None)

    def __call__(self, X, out=None, stream=None):
        M = X.shape[0]
        send, y_local = local_buffer(M, self.bounds, self.rank, X.device)
        if self.lin is not None and M:
            self.lin(X, out=y_local, stream=stream)
            if stream is not None and hasattr(stream, "cuda_stream"):
                torch.cuda.current_stream().wait_stream(stream)  # the exchange runs on the current stream
        return gather_columns(send, M, self.bounds, out, self.active, self.group)

    def free(self):
        if self.lin is not None:
            self.lin.free()
            self.lin = None
