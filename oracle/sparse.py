"""Sparse attention with branch-consistent indexer groups over a proposal tree
(oracle; test infrastructure only).

Source: "SpecOPD: Branch-Parallel On-Policy Distillation for Speculative
Decoding" as listed on thelatestinai.com, Fig 4:
  * every row reuses the complete trunk group keys, including the group that
    ends at the anchor's last complete boundary;
  * an incomplete boundary group stays in the row's causal tail;
  * a group completed by branch tokens needs a branch-specific indexer group
    key;
  * indexer queries select eligible complete groups with top-k; attention
    reads the selected groups' keys and values plus the causal tail, which
    bypasses top-k.

Readings where the pages are silent (plainest choice):
  * groups are g consecutive semantic positions of the row's own history
    (trunk through the anchor, then the branch's tokens): group m covers
    positions m g .. m g + g - 1; it is complete for a row at position p when
    m g + g - 1 <= p, and the causal tail is the row's own incomplete group,
    positions floor((p + 1) / g) g .. p (empty when p + 1 is a multiple of g);
  * a group's indexer key is the mean of its members' indexer keys; a row's
    score for a group is its indexer query dotted with that key; selection is
    per KV head (the query heads of a GQA group share it), the k highest
    scores, ties to the earlier group; with k or fewer complete groups all are
    selected;
  * attention itself is the tree attention of attention.py (rotate-half RoPE
    at semantic positions, scale 1/sqrt(d)) restricted to the selected groups'
    members and the tail.

Written from these definitions in fp64, one row at a time, with no blocking
or reuse of group keys across rows.
"""
from __future__ import annotations

from typing import Iterable, List, Mapping, Optional, Sequence, Tuple

import numpy as np

from . import attention as _attn
from . import tree as _tree


def history(pt: _tree.PackedTrees, r: int) -> List[int]:
    """Packed rows of r's history in position order (root first, r last)."""
    return _tree.ancestors(pt, r)[::-1] + [r]


def group_scores(pt: _tree.PackedTrees, r: int, qi: np.ndarray, ki: np.ndarray, g: int,
                 kvh: int) -> np.ndarray:
    """fp64 indexer scores of row r's complete groups for KV head kvh: group m's
    key is the mean of the indexer keys of history positions m g .. m g + g - 1
    (branch-specific when the group holds branch tokens, since the history is
    the branch's own), and its score is the row's indexer query dotted with it."""
    hist = history(pt, r)
    n_complete = len(hist) // g
    if n_complete == 0:
        return np.zeros(0)
    keys = np.stack([np.mean(np.asarray(ki[hist[m * g:(m + 1) * g], kvh], dtype=np.float64), axis=0)
                     for m in range(n_complete)])
    return keys @ np.asarray(qi[r, kvh], dtype=np.float64)


def top_groups(scores: np.ndarray, topk: int) -> List[int]:
    """The topk highest scores (ties to the earlier group), ascending; all
    groups when there are topk or fewer."""
    order = sorted(range(len(scores)), key=lambda m: (-scores[m], m))
    return sorted(order[:topk])


def selected_columns(pt: _tree.PackedTrees, r: int, qi: np.ndarray, ki: np.ndarray, g: int, topk: int,
                     kvh: int, groups: Optional[Sequence[int]] = None) -> List[int]:
    """Packed columns row r attends to for KV head kvh: the members of its
    top-k complete groups (by fp64 indexer score), or of the given `groups`,
    followed by its causal tail."""
    hist = history(pt, r)
    p = len(hist) - 1
    n_complete = (p + 1) // g
    tail = hist[n_complete * g:]
    if n_complete == 0:
        return tail
    chosen = top_groups(group_scores(pt, r, qi, ki, g, kvh), topk) if groups is None else sorted(groups)
    cols = [c for m in chosen for c in hist[m * g:(m + 1) * g]]
    return cols + tail


def sparse_tree_attention(pt: _tree.PackedTrees, q: np.ndarray, k: np.ndarray, v: np.ndarray, qi: np.ndarray,
                          ki: np.ndarray, g: int, topk: int, theta: float, scale: Optional[float] = None,
                          rows: Optional[Iterable[int]] = None,
                          selections: Optional[Mapping[Tuple[int, int], Sequence[int]]] = None) -> np.ndarray:
    """O[r, h] over the selected columns of row r for KV head h // (Hq / Hkv).
    q [N, Hq, d], k/v [N, Hkv, d] (RoPE applied here at semantic positions),
    qi/ki [N, Hkv, di] indexer features.  Returns [len(rows), Hq, d], fp64.
    `selections` maps (row, kvh) to a group list used instead of the fp64
    top-k (a selection shown elsewhere to be a valid top-k)."""
    if g < 1 or topk < 1:
        raise ValueError("group size and top-k must be positive")
    N, Hq, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    pos = _tree.positions(pt)
    qr = _attn.rope(q, pos, theta)
    kr = _attn.rope(k, pos, theta)
    vv = np.asarray(v, dtype=np.float64)
    rows = list(range(N)) if rows is None else list(rows)
    out = np.zeros((len(rows), Hq, d))
    for n, r in enumerate(rows):
        for kvh in range(Hkv):
            given = None if selections is None else selections.get((r, kvh))
            cols = selected_columns(pt, r, qi, ki, g, topk, kvh, given)
            for h in range(kvh * G, (kvh + 1) * G):
                out[n, h] = _attn._softmax_attend(qr[r, h], kr[cols, kvh], vv[cols, kvh], scale)
    return out
