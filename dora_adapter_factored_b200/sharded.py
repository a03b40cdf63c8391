"""Sharding the factored norm across devices.

* d_in sharding ("Scaling DoRA ...", section 6: a base weight sharded
  FSDP2-style needs chunk-wise partial sums followed by an all-reduce;
  section 2: every term of the squared row norm is a sum over the columns of
  W0) -- ``column_shard``, ``sharded_factored_norm`` below;
* row sharding: rows are independent, so each rank takes a contiguous block of
  output rows of W0 and B (``row_shard``) and ``all_gather_rows`` replicates n;
* module sharding of a grouped call: whole modules per rank, balanced by
  FLOPs (``module_shard``), no collective at all.

Each rank holds a contiguous column shard of W0 and A (the same columns of
both) and all of B.  It computes its shard's squared row-norm contribution on
its GPU (``dora_factored_norm_sq``), one all-reduce (sum) of the d_out fp32
values combines the shards over ``torch.distributed`` (NCCL over NVLink on
GPUs), and ``dora_norm_finalize`` takes the square root and forms g.  Only
d_out floats cross the interconnect, whatever d_in and r.
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

import torch
import torch.distributed as dist

from ._abi import dora_factored_norm_sq, dora_norm_finalize


def column_shard(d_in: int, rank: int, world: int, align: int = 64) -> Tuple[int, int]:
    """[begin, end) of rank's columns: contiguous, in rank order, boundaries on
    multiples of ``align`` (whole 64-column k-blocks of the norm GEMM), the
    remainder going to the last ranks.  Shards may be empty when d_in is small."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    if d_in < 0 or align < 1:
        raise ValueError("d_in must be >= 0 and align >= 1")
    blocks = -(-d_in // align)
    b0 = rank * blocks // world
    b1 = (rank + 1) * blocks // world
    return min(b0 * align, d_in), min(b1 * align, d_in)


def all_reduce_rows(sq: torch.Tensor, group=None) -> torch.Tensor:
    """Sums the per-rank squared partials in place (one all-reduce of d_out
    floats over ``group``); a no-op when no process group is initialised."""
    if dist.is_available() and dist.is_initialized():
        dist.all_reduce(sq, op=dist.ReduceOp.SUM, group=group)
    return sq


def sharded_factored_norm(W0_shard: torch.Tensor, A_shard: torch.Tensor, B: torch.Tensor,
                          s: float, m: Optional[torch.Tensor] = None, eps: float = 0.0,
                          group=None):
    """Row norm n of W0 + s B A (and g = m / max(n, eps) when m is given) from
    this rank's column shard of W0 and A.  Every rank of ``group`` calls it
    with its own shard; all get the same n (and g).  Runs on the current CUDA
    stream, which the all-reduce also orders against.  Returns (n, g or None)."""
    if W0_shard.shape[1] == 0:
        sq = torch.zeros(W0_shard.shape[0], dtype=torch.float32, device=W0_shard.device)
    else:
        sq = dora_factored_norm_sq(W0_shard, A_shard, B, s)
    all_reduce_rows(sq, group)
    return dora_norm_finalize(sq, m, eps, n_out=sq)


def row_shard(d_out: int, rank: int, world: int, align: int = 128) -> Tuple[int, int]:
    """[begin, end) of rank's output rows: contiguous, in rank order, on
    multiples of ``align`` (whole 128-row tiles of the norm GEMM)."""
    return column_shard(d_out, rank, world, align)


def all_gather_rows(n_local: torch.Tensor, d_out: int, group=None, align: int = 128) -> torch.Tensor:
    """The full [d_out] vector from every rank's ``row_shard`` slice (one
    all-gather of equal-sized padded slices); n_local itself without a
    process group."""
    if not (dist.is_available() and dist.is_initialized()):
        return n_local
    world = dist.get_world_size(group)
    bounds = [row_shard(d_out, r, world, align) for r in range(world)]
    width = max(b - a for a, b in bounds)
    padded = torch.zeros(width, dtype=n_local.dtype, device=n_local.device)
    padded[: n_local.numel()] = n_local
    parts = [torch.empty_like(padded) for _ in range(world)]
    dist.all_gather(parts, padded, group=group)
    return torch.cat([parts[r][: b - a] for r, (a, b) in enumerate(bounds)])


def module_shard(flops: Sequence[float], world: int) -> List[List[int]]:
    """Modules of a grouped call per rank: largest first, each to the rank with
    the least work so far (ties: lower rank), each rank's list in module order.
    Deterministic; the heaviest rank carries at most the mean plus one module."""
    if world < 1:
        raise ValueError("world must be >= 1")
    load = [0.0] * world
    owner = [0] * len(flops)
    for i in sorted(range(len(flops)), key=lambda k: (-flops[k], k)):
        r = min(range(world), key=lambda q: (load[q], q))
        owner[i] = r
        load[r] += flops[i]
    return [[i for i in range(len(flops)) if owner[i] == r] for r in range(world)]
