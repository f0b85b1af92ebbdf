"""Data-parallel plumbing for the ELSAA operator across ranks.

The (batch, head) units of the operator are independent, so ranks shard the
batch with no exchange in the data path.  The gate weights and lambda are
shared by every unit: their gradients are sums over all tokens of all ranks,
which takes one all-reduce of 2 d + 3 values per step.  Works on any
torch.distributed backend (NCCL on GPUs, gloo on the CPU).
"""

from __future__ import annotations

from typing import Sequence

import torch
import torch.distributed as dist


def rank_seed(base_seed: int, rank: int) -> int:
    """Seed of the synthetic batch a rank draws: every rank gets its own data."""
    return base_seed + rank


def allreduce_param_grads(dgate_w: torch.Tensor, dgate_b: torch.Tensor,
                          dlam: torch.Tensor) -> None:
    """Sum the shared-parameter gradients over ranks, in place, with one
    all-reduce of a packed [2 d + 3] buffer."""
    flat = torch.cat([dgate_w.reshape(-1), dgate_b.reshape(-1), dlam.reshape(-1)])
    dist.all_reduce(flat, op=dist.ReduceOp.SUM)
    n, m = dgate_w.numel(), dgate_b.numel()
    dgate_w.view(-1).copy_(flat[:n])
    dgate_b.view(-1).copy_(flat[n:n + m])
    dlam.view(-1).copy_(flat[n + m:])


def max_over_ranks(values: Sequence[float], device) -> list:
    """Element-wise maximum of per-rank timings (the slowest rank sets the time)."""
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()
