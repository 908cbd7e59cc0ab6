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

from typing import Iterable, List, Optional

import numpy as np

from . import attention as _attn
from . import tree as _tree


def history(pt: _tree.PackedTrees, r: int) -> List[int]:
    """Packed rows of r's history in position order (root first, r last)."""
    return _tree.ancestors(pt, r)[::-1] + [r]


def _scores_fp32(qr: np.ndarray, members: List[np.ndarray]) -> np.ndarray:
    """Indexer scores taken in fp32 in a fixed order: each group key is the
    sequential fp32 sum of its members' keys divided by g, each score a
    sequential chain of fused multiply-adds over the key's elements (every step
    rounded once to fp32)."""
    out = np.zeros(len(members))
    q32 = np.asarray(qr, dtype=np.float32)
    for m, mem in enumerate(members):
        key = np.zeros(mem.shape[1], dtype=np.float32)
        for row in np.asarray(mem, dtype=np.float32):
            key = (key + row).astype(np.float32)
        key = (key / np.float32(mem.shape[0])).astype(np.float32)
        acc = np.float32(0.0)
        for e in range(key.shape[0]):
            acc = np.float32(float(q32[e]) * float(key[e]) + float(acc))
        out[m] = float(acc)
    return out


def selected_columns(pt: _tree.PackedTrees, r: int, qi: np.ndarray, ki: np.ndarray, g: int, topk: int,
                     kvh: int, decide_fp32: bool = False) -> List[int]:
    """Packed columns row r attends to for KV head kvh: the members of its
    top-k complete groups (by indexer score) and its causal tail.  With
    decide_fp32 the scores that decide the selection are taken in fp32 (see
    _scores_fp32) rather than fp64."""
    hist = history(pt, r)
    p = len(hist) - 1
    n_complete = (p + 1) // g
    tail = hist[n_complete * g:]
    if n_complete == 0:
        return tail
    if decide_fp32:
        scores = _scores_fp32(qi[r, kvh], [ki[hist[m * g:(m + 1) * g], kvh] for m in range(n_complete)])
    else:
        keys = np.stack([np.mean(np.asarray(ki[hist[m * g:(m + 1) * g], kvh], dtype=np.float64), axis=0)
                         for m in range(n_complete)])
        scores = keys @ np.asarray(qi[r, kvh], dtype=np.float64)
    order = sorted(range(n_complete), key=lambda m: (-scores[m], m))
    chosen = sorted(order[:topk])
    cols = [c for m in chosen for c in hist[m * g:(m + 1) * g]]
    return cols + tail


def sparse_tree_attention(pt: _tree.PackedTrees, q: np.ndarray, k: np.ndarray, v: np.ndarray, qi: np.ndarray,
                          ki: np.ndarray, g: int, topk: int, theta: float, scale: Optional[float] = None,
                          rows: Optional[Iterable[int]] = None, decide_fp32: bool = False) -> np.ndarray:
    """O[r, h] over the selected columns of row r for KV head h // (Hq / Hkv).
    q [N, Hq, d], k/v [N, Hkv, d] (RoPE applied here at semantic positions),
    qi/ki [N, Hkv, di] indexer features.  Returns [len(rows), Hq, d].  The
    attention is fp64; decide_fp32 takes only the selection's scores in fp32,
    the precision in which a GPU kernel makes that integer decision."""
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
            cols = selected_columns(pt, r, qi, ki, g, topk, kvh, decide_fp32)
            for h in range(kvh * G, (kvh + 1) * G):
                out[n, h] = _attn._softmax_attend(qr[r, h], kr[cols, kvh], vv[cols, kvh], scale)
    return out
