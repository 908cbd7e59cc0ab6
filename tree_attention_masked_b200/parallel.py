"""Host logic for running the scoring step on several GPUs, one process per GPU.

The trees of a batch are independent problems (SpecOPD, Fig 3: each proposal
tree is packed and scored on its own), so ranks never exchange data inside a
step.  The only cross-rank quantities are:

* the slowest rank's step time (the job is as fast as its slowest rank);
* the E2E-TV loss when one logical batch of branches is split over ranks.
  The daiwk.github.io write-up, section "Equations", normalises L by the total
  number of supervised predictions, L = 1 - (1/count) sum_b sum_j prod_{i<=j}
  alpha_{b,i}.  A rank that scores its own branches with the global `count`
  returns L_r = 1 - (1/count) * (its part of the double sum), and its
  gradient rows are already the global gradient's rows.  The global loss is
  then sum_r L_r - (world - 1).

Every function takes an optional process group and works with any
torch.distributed backend (NCCL on the GPUs, gloo in the CPU tests).
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch
import torch.distributed as dist


def shard_range(n: int, world: int, rank: int) -> Tuple[int, int]:
    """[lo, hi) of a contiguous split of n items over `world` ranks; the first
    n % world ranks take one item more."""
    if world < 1 or not 0 <= rank < world or n < 0:
        raise ValueError(f"bad split: n={n} world={world} rank={rank}")
    base, extra = divmod(n, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def _world(group) -> int:
    return dist.get_world_size(group) if dist.is_initialized() else 1


def global_count(local_count: int, group=None, device: Optional[torch.device] = None) -> int:
    """Total number of supervised predictions over all ranks."""
    if _world(group) == 1:
        return int(local_count)
    t = torch.tensor([float(local_count)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
    return int(round(t.item()))


def global_loss(local_loss: float, group=None, device: Optional[torch.device] = None) -> float:
    """Recombine per-rank E2E-TV losses computed with the global count."""
    world = _world(group)
    if world == 1:
        return float(local_loss)
    t = torch.tensor([float(local_loss)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
    return t.item() - (world - 1)


def max_time_ms(local_ms: float, group=None, device: Optional[torch.device] = None) -> float:
    """Slowest rank's time (device-timed on each rank)."""
    if _world(group) == 1:
        return float(local_ms)
    t = torch.tensor([float(local_ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return t.item()
