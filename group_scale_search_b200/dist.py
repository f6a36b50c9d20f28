"""Multi-GPU plumbing for the group-scale search path (one process per GPU,
torch.distributed: NCCL on GPUs, gloo on CPU for tests).

The search, RTN, packing, dequantization and proxy error act on independent
groups, so GPUs split the work (whole matrices, or row ranges of one matrix)
and exchange nothing.  The exchanges are small and only arise when one
matrix or one calibration set is split: token-sharded calibration (every
rank sums x^2 over its own tokens with tq_imatrix(alpha = 1) and an
all-reduce adds the partial sums before the division by the total token
count), and a row-sharded matrix's proxy error (an all-reduce of the
per-matrix fp64 (num, den) pairs before the ratio).  The same two hold for the
full-Hessian path: H = sum_t x_t^T x_t adds over token shards (every rank
runs tq_hessian on its tokens, an all-reduce adds the fp64 copies), after
which the GPTQ/LDLQ sweep splits the rows of W with no exchange (rows are
independent given the factor of H^-1); and tr(E H E^T) = ||X E^T||^2 adds
over token shards and over row shards, so tq_proxy_error_full's (num, den)
go through allreduce_proxy.
"""
from __future__ import annotations

import datetime
from typing import List, Optional, Sequence, Tuple

import torch
import torch.distributed as dist

__all__ = ["shard_range", "shard_units", "allreduce_imatrix", "allreduce_hessian", "allreduce_proxy",
           "max_over_ranks", "init_from_env"]


def shard_range(n: int, rank: int, world: int) -> Tuple[int, int]:
    """Contiguous share [start, end) of n items for `rank`; sizes differ by at most one."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"bad rank {rank} of world {world}")
    base, extra = divmod(n, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def shard_units(costs: Sequence[float], world: int) -> List[List[int]]:
    """Assigns units (e.g. the linears of a layer) to ranks, largest first to
    the least loaded rank, so per-rank work is balanced.  Every unit goes to
    exactly one rank; ties go to the lower rank."""
    load = [0.0] * world
    plan: List[List[int]] = [[] for _ in range(world)]
    for i in sorted(range(len(costs)), key=lambda k: (-costs[k], k)):
        r = min(range(world), key=lambda q: (load[q], q))
        plan[r].append(i)
        load[r] += costs[i]
    return [sorted(p) for p in plan]


def allreduce_imatrix(local_sums: torch.Tensor, total_tokens: int, group=None) -> torch.Tensor:
    """m = (sum over ranks of the per-column sums of x^2) / total_tokens.

    local_sums: this rank's sum_t x_{t,j}^2 over its tokens (fp32, e.g. from
    tq_imatrix(X_local, alpha=1)).  The reduction runs in fp64 so the result
    does not depend on the number of ranks beyond fp64 rounding."""
    if total_tokens <= 0:
        raise ValueError("total_tokens must be positive")
    acc = local_sums.to(torch.float64)
    if dist.is_available() and dist.is_initialized():
        dist.all_reduce(acc, op=dist.ReduceOp.SUM, group=group)
    return (acc / float(total_tokens)).to(torch.float32)


def allreduce_hessian(local_h: torch.Tensor, group=None) -> torch.Tensor:
    """H = sum over ranks of X_r^T X_r for token-sharded calibration.

    local_h: this rank's Hessian of its own tokens (fp32 from tq_hessian, or
    fp64); the sum runs in fp64 so it does not depend on the rank count beyond
    fp64 rounding, and the fp64 result is what the factorisation of H^-1 for
    the GPTQ sweep wants.  Every rank gets the whole H."""
    acc = local_h.to(torch.float64)
    if dist.is_available() and dist.is_initialized():
        dist.all_reduce(acc, op=dist.ReduceOp.SUM, group=group)
    return acc


def allreduce_proxy(num: torch.Tensor, den: torch.Tensor, group=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Proxy error of matrices whose rows (or, for tq_proxy_error_full, whose
    calibration tokens) are split over ranks: every rank passes its fp64
    (num, den); the sums over ranks are the whole matrices' tr(E H E^T) and
    tr(W H W^T) (the ratio is taken after the sum, never averaged over
    ranks)."""
    if num.dtype != torch.float64 or den.dtype != torch.float64:
        raise ValueError("num and den must be float64")
    both = torch.stack([num, den])
    if dist.is_available() and dist.is_initialized():
        dist.all_reduce(both, op=dist.ReduceOp.SUM, group=group)
    return both[0], both[1]


def max_over_ranks(value: float, device: Optional[torch.device] = None, group=None) -> float:
    """The maximum of `value` over all ranks (how every multi-GPU time is reported)."""
    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


def init_from_env(backend: str = "nccl", timeout_s: float = 120.0) -> Tuple[int, int, int]:
    """Initialises the default process group from torchrun's environment
    (RANK, LOCAL_RANK, WORLD_SIZE, MASTER_ADDR/PORT) with a finite timeout, so
    ranks waiting on a rank that died end with an error instead of hanging.
    Returns (world, rank, local_rank); a single process is world 1."""
    import os
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and not dist.is_initialized():
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return world, rank, local
