"""Host-side helpers for one-process-per-GPU runs (torch.distributed).

The MX cast and GEMM work on independent blocks and tiles, so multi-GPU runs
shard whole problems (or whole rows of one problem) across ranks with no
data-path collective.  These helpers only split work and reduce timings; they
run unchanged under NCCL (one GPU per rank) and gloo (CPU tests).
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def world() -> tuple[int, int]:
    if dist.is_available() and dist.is_initialized():
        return dist.get_rank(), dist.get_world_size()
    return 0, 1


def shard_rows(rows: int, world_size: int, rank: int, multiple: int = 1) -> tuple[int, int]:
    """Contiguous [start, stop) row range of `rank`; boundaries are multiples of
    `multiple` (32 when rows are the block axis), the last rank takes the tail."""
    units = (rows + multiple - 1) // multiple
    per = units // world_size
    extra = units % world_size
    start_u = rank * per + min(rank, extra)
    stop_u = start_u + per + (1 if rank < extra else 0)
    return min(start_u * multiple, rows), min(stop_u * multiple, rows)


def max_over_ranks(x: float, device: torch.device | None = None) -> float:
    """The slowest rank's value (timings are reported as the max over ranks)."""
    rank, ws = world()
    if ws == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier() -> None:
    rank, ws = world()
    if ws > 1:
        dist.barrier()
