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


# ---------------------------------------------------------------------------
# Data-parallel weight gradient: tokens are sharded across ranks.
#
# dW = alpha * dY^T X contracts over the tokens, so a rank that holds tokens
# [t0, t1) of dY (T x D_out) and X (T x D_in) computes a partial dW over its
# tokens and the ranks sum the partials: the one exchange on this path, an
# all-reduce (every rank gets dW) or a reduce-scatter (rank r gets rows
# [r D_out / W, (r + 1) D_out / W) of dW), over NCCL between GPUs.  The casts
# along tokens (fixed-sign Hadamard + stochastic rounding, "Format-Aware
# Fusion for Fast FP4 Pretraining", abstract) are sharded casts: each rank's
# codes are exactly its slice of the whole tensor's codes, so the summed dW is
# the unsharded one up to the order of the fp32 sums.
# ---------------------------------------------------------------------------

class CudaOps:
    """The sharded cast and the GEMM on this rank's GPU (libmx kernels)."""

    @staticmethod
    def cast(t, fmt, seed, sign_mask, shard):
        from . import mx
        return mx.quantize(t, 0, fmt, rnd="sr", seed=seed, hadamard=True, sign_mask=sign_mask, shard=shard)

    @staticmethod
    def gemm(ac, as_, bc, bs, M, N, K, fmt, alpha):
        from . import mx
        return mx.gemm(ac, as_, bc, bs, M, N, K, fa=fmt, alpha=alpha, out_dtype=torch.float32)


def token_shards(tokens: int, world_size: int, multiple: int = 256) -> list[tuple[int, int]]:
    """Contiguous token ranges, one per rank, on `multiple`-token boundaries
    (256 keeps every partial GEMM's K a multiple of the FP4 MMA's K step)."""
    if tokens % multiple != 0:
        raise ValueError(f"tokens ({tokens}) must be a multiple of {multiple}")
    return [shard_rows(tokens, world_size, r, multiple) for r in range(world_size)]


def wgrad(dy_local, x_local, t0: int, total_tokens: int, *, fmt: str = "e2m1", seed_dy: int = 42,
          seed_x: int = 43, sign_mask: int = 0x6A09E667, reduce: str = "all_reduce", ops=CudaOps):
    """dW = (1/32) (H D dY)^T (H D X) over all ranks' tokens, from this rank's
    token shard (tokens [t0, t0 + len) of total_tokens).

    Returns the full fp32 dW (D_out x D_in) with reduce="all_reduce", or this
    rank's row block of it with reduce="reduce_scatter" (D_out must then be a
    multiple of the world size).  `ops` supplies the cast and the GEMM (the
    CUDA kernels by default)."""
    rank, ws = world()
    tl, d_out = dy_local.shape
    d_in = x_local.shape[1]
    if x_local.shape[0] != tl:
        raise ValueError("dY and X shards must hold the same tokens")
    ac, as_ = ops.cast(dy_local, fmt, seed_dy, sign_mask, (t0, 0, total_tokens, d_out))
    bc, bs = ops.cast(x_local, fmt, seed_x, sign_mask, (t0, 0, total_tokens, d_in))
    part = ops.gemm(ac, as_, bc, bs, d_out, d_in, tl, fmt, 1.0 / 32)
    if ws == 1:
        return part
    if reduce == "all_reduce":
        dist.all_reduce(part, op=dist.ReduceOp.SUM)
        return part
    if reduce == "reduce_scatter":
        if d_out % ws != 0:
            raise ValueError("reduce_scatter needs D_out divisible by the world size")
        out = torch.empty((d_out // ws, d_in), dtype=part.dtype, device=part.device)
        dist.reduce_scatter_tensor(out, part.contiguous(), op=dist.ReduceOp.SUM)
        return out
    raise ValueError(f"unknown reduce {reduce!r}")
