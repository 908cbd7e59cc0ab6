"""Host logic for running the scoring step on several GPUs, one process per GPU.

One logical batch of proposal trees is split over the ranks:

* attention by query rows: each rank scores a contiguous run of the packed
  128-row query tiles, the runs balanced by visible (row, column) pairs (a
  trunk tile's cost grows with its position; a branch row sees its anchor's
  prefix plus its own samples).  Every rank holds the keys and values its
  tiles see; no data moves between ranks;
* the overlap, E2E-TV loss and gradient by whole branches (all W rows of a
  branch on one rank, since its prefix products couple them).

The only cross-rank quantities are:

* the slowest rank's step time (the job is as fast as its slowest rank);
* the E2E-TV loss of the split batch of branches.
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

from typing import List, Optional, Sequence, Tuple

import numpy as np
import torch
import torch.distributed as dist

TILE_ROWS = 128


def shard_range(n: int, world: int, rank: int) -> Tuple[int, int]:
    """[lo, hi) of a contiguous split of n items over `world` ranks; the first
    n % world ranks take one item more."""
    if world < 1 or not 0 <= rank < world or n < 0:
        raise ValueError(f"bad split: n={n} world={world} rank={rank}")
    base, extra = divmod(n, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def tile_costs(trunk_len: Sequence[int], num_branches: Sequence[int], anchors: np.ndarray, W: int,
               pack_terminal: bool = True) -> np.ndarray:
    """Visible (row, column) pairs of every packed 128-row query tile, in the
    packing order of specopd_build_tree_mask (per tree: trunk, then each
    branch's samples; tiles never straddle two trees).  Trunk row j sees j + 1
    columns; sample i of a branch at anchor a sees a + 1 trunk columns and its
    own samples 1..i."""
    rpb = W if pack_terminal else W - 1
    out: List[np.ndarray] = []
    a_off = 0
    for T, B in zip(trunk_len, num_branches):
        anc = np.asarray(anchors[a_off:a_off + B], dtype=np.int64)
        a_off += B
        per_row = np.concatenate([np.arange(1, T + 1, dtype=np.int64),
                                  (anc[:, None] + 1 + np.arange(1, rpb + 1)[None, :]).reshape(-1)])
        n = per_row.shape[0]
        pad = (-n) % TILE_ROWS
        out.append(np.concatenate([per_row, np.zeros(pad, np.int64)]).reshape(-1, TILE_ROWS).sum(axis=1))
    return np.concatenate(out) if out else np.zeros(0, np.int64)


def tile_rows(trunk_len: Sequence[int], num_branches: Sequence[int], W: int, pack_terminal: bool = True) -> np.ndarray:
    """[first row, one past the last row] of every packed query tile, in the
    order of tile_costs."""
    rpb = W if pack_terminal else W - 1
    out = []
    base = 0
    for T, B in zip(trunk_len, num_branches):
        n = T + B * rpb
        for r in range(base, base + n, TILE_ROWS):
            out.append((r, min(base + n, r + TILE_ROWS)))
        base += n
    return np.asarray(out, dtype=np.int64).reshape(-1, 2)


def split_tiles(costs: np.ndarray, world: int, rank: int) -> Tuple[int, int]:
    """[t0, t1) of a contiguous split of the tiles over `world` ranks with about
    equal cost: rank r ends at the first tile whose running cost reaches
    (r + 1) / world of the total (the last rank takes the rest)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"bad split: world={world} rank={rank}")
    n = int(costs.shape[0])
    cum = np.cumsum(costs, dtype=np.float64)
    total = cum[-1] if n else 0.0

    def end(r):
        if r >= world - 1:
            return n
        return min(n, int(np.searchsorted(cum, total * (r + 1) / world, side="left")) + 1)

    t0 = 0 if rank == 0 else end(rank - 1)
    return min(t0, n), max(min(end(rank), n), min(t0, n))


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


# ---------------------------------------------------------------- vocabulary-parallel LM head
def vocab_range(V: int, world: int, rank: int, align: int = 256) -> Tuple[int, int]:
    """[v0, v1) of a contiguous split of the vocabulary over `world` ranks in
    blocks of `align` entries (the LM-head tile width; a shard's gradient
    columns then start on 16-byte boundaries); the last rank ends at V."""
    blocks = (V + align - 1) // align
    b0, b1 = shard_range(blocks, world, rank)
    return min(V, b0 * align), min(V, b1 * align)


def gather_rows(x: torch.Tensor, group=None) -> torch.Tensor:
    """Every rank's [n] tensor stacked in rank order: [world, n] (the tensor
    itself, unsqueezed, on one rank)."""
    world = _world(group)
    if world == 1:
        return x.unsqueeze(0)
    parts = [torch.empty_like(x) for _ in range(world)]
    dist.all_gather(parts, x.contiguous(), group=group)
    return torch.stack(parts)


def lm_head_vocab_parallel(h_draft, head_draft_shard, h_teacher, head_teacher_shard, num_branches: int, W: int,
                           grad_shard, workspace, status, group=None, stream=None):
    """The LM head + overlap with the vocabulary split over the ranks of
    `group` (each rank holds all hidden states and its rows of both heads):
    phase 0, a gather and merge of the per-row log-sum-exps, phase 1, a gather
    and merge of the alpha / q_less shares, the E2E-TV loss on the merged
    alpha (every rank), phase 2 for the rank's gradient columns.  Three per-row
    exchanges; every merge is the library's, in rank order, so every rank gets
    identical alpha, L and dL/dalpha.  Returns (alpha, q_less, loss, grad_alpha)."""
    from . import specopd as S
    R = h_draft.shape[0]
    dev = h_draft.device
    f = lambda: torch.empty(R, device=dev, dtype=torch.float32)
    lz_l, lt_l = f(), f()
    S.specopd_lm_head_shard_phase(0, h_draft, head_draft_shard, h_teacher, head_teacher_shard, workspace, status,
                                  lz_l, lt_l, stream=stream)
    lz2, lt2 = f(), f()
    S.specopd_merge_parts(gather_rows(lz_l, group), 1, lz2, stream=stream)
    S.specopd_merge_parts(gather_rows(lt_l, group), 1, lt2, stream=stream)
    a_l, q_l = f(), f()
    S.specopd_lm_head_shard_phase(1, h_draft, head_draft_shard, h_teacher, head_teacher_shard, workspace, status,
                                  a_l, q_l, lz2=lz2, lt2=lt2, stream=stream)
    alpha, q_less = f(), f()
    S.specopd_merge_parts(gather_rows(a_l, group), 0, alpha, stream=stream)
    S.specopd_merge_parts(gather_rows(q_l, group), 0, q_less, stream=stream)
    loss, g = torch.empty(1, device=dev, dtype=torch.float32), f()
    S.specopd_e2e_tv_loss(alpha, num_branches, W, 0.0, loss, g, stream=stream)
    if grad_shard is not None:
        S.specopd_lm_head_shard_phase(2, h_draft, head_draft_shard, h_teacher, head_teacher_shard, workspace, status,
                                      grad_shard, lz2=lz2, q_less=q_less, grad_alpha=g, stream=stream)
    return alpha, q_less, loss, g
