"""Proposal-tree packing and visibility (oracle; test infrastructure only).

Definitions followed (SpecOPD, thelatestinai.com listing):
  * Fig 2 step 3: sampled continuations are attached to their anchors, giving a
    shared reference trunk and separate draft branches.
  * Fig 3: the tree mask restricts each packed row to itself and its ancestors;
    rows and columns share one packed-token order.
  * daiwk.github.io write-up, section "Equations": the history of sample
    y_{b,i} is (x_{<=a_b}, y_{b,<i}); the anchor row predicts the first sample,
    the row of y_{b,i-1} predicts y_{b,i}; semantic positions are a_b + i.
  * same write-up, section "Inputs and code mapping": anchors are zero-based;
    the tree is built from the reference length, the anchors and the width.

Packing (the pages leave the order open; this is the plainest reading): each
tree is the trunk 0..T-1 followed by its branches in caller order, each branch
y_{b,1..} contiguous; trees are concatenated and never see each other.
With ``pack_terminal`` the terminal sample y_{b,W} also gets a row (its row
is scored but never read out); without it a branch has W-1 rows, as in Fig 3.

Everything here is derived by walking parent pointers: positions are depths,
visibility is the ancestor set.  The compact fields the CUDA path emits
(trunk limit, branch id, ancestor bits, prediction rows) are then read off
those sets, not from closed forms.
"""
from __future__ import annotations

import dataclasses
from typing import List, Sequence

import numpy as np


class TreeError(ValueError):
    pass


@dataclasses.dataclass
class PackedTrees:
    cu_rows: np.ndarray      # int64 [num_trees+1] first packed row of each tree
    parent: np.ndarray       # int64 [N] packed parent row, -1 at each tree's root
    tree_of: np.ndarray      # int64 [N]
    is_trunk: np.ndarray     # bool  [N]
    trunk_index: np.ndarray  # int64 [N] tree-local trunk index, -1 for branch rows
    branch_of: np.ndarray    # int64 [N] global branch id, -1 for trunk rows
    sample_index: np.ndarray # int64 [N] i of y_{b,i} (1-based), 0 for trunk rows
    branch_rows: List[List[int]]  # per global branch: packed rows of y_{b,1..}
    anchors_global: np.ndarray    # int64 [sum B] packed row of each anchor
    W: int
    pack_terminal: bool

    @property
    def num_rows(self) -> int:
        return int(self.parent.shape[0])


def pack(trunk_len: Sequence[int], prompt_len: Sequence[int], num_branches: Sequence[int],
         anchors: Sequence[int], W: int, pack_terminal: bool = True) -> PackedTrees:
    """Lay out the trees and set parent pointers (trunk j -> j-1; y_{b,1} -> a_b;
    y_{b,i} -> y_{b,i-1})."""
    anchors = np.asarray(anchors, dtype=np.int64)
    if W < 1 or W > 64:
        raise TreeError("branch width W must be in [1, 64]")
    if not (len(trunk_len) == len(prompt_len) == len(num_branches)):
        raise TreeError("per-tree arrays differ in length")
    if anchors.shape[0] != int(sum(num_branches)):
        raise TreeError("need one anchor per branch")
    rpb = W if pack_terminal else W - 1
    parent, tree_of, is_trunk, tidx, bof, sidx = [], [], [], [], [], []
    cu = [0]
    branch_rows: List[List[int]] = []
    anc_g = []
    a_off = 0
    gb = 0
    for t, (T, P, B) in enumerate(zip(trunk_len, prompt_len, num_branches)):
        T, P, B = int(T), int(P), int(B)
        if T < 1 or P < 0 or P > T - 1 or B < 0:
            raise TreeError(f"tree {t}: need T >= 1, 0 <= P <= T-1, B >= 0")
        base = cu[-1]
        for j in range(T):
            parent.append(base + j - 1 if j > 0 else -1)
            tree_of.append(t); is_trunk.append(True); tidx.append(j); bof.append(-1); sidx.append(0)
        for b in range(B):
            a = int(anchors[a_off + b])
            if a < P or a > T - 1:
                raise TreeError(f"tree {t} branch {b}: anchor {a} outside reference positions [{P}, {T - 1}]")
            anc_g.append(base + a)
            rows = []
            for i in range(1, rpb + 1):
                r = len(parent)
                parent.append(base + a if i == 1 else r - 1)
                tree_of.append(t); is_trunk.append(False); tidx.append(-1); bof.append(gb); sidx.append(i)
                rows.append(r)
            branch_rows.append(rows)
            gb += 1
        a_off += B
        cu.append(len(parent))
    return PackedTrees(np.asarray(cu, np.int64), np.asarray(parent, np.int64),
                       np.asarray(tree_of, np.int64), np.asarray(is_trunk, bool),
                       np.asarray(tidx, np.int64), np.asarray(bof, np.int64),
                       np.asarray(sidx, np.int64), branch_rows,
                       np.asarray(anc_g, np.int64), W, pack_terminal)


def ancestors(pt: PackedTrees, r: int) -> List[int]:
    """Strict ancestors of packed row r, nearest first (walk of parent pointers)."""
    out = []
    p = int(pt.parent[r])
    while p >= 0:
        out.append(p)
        p = int(pt.parent[p])
    return out


def visible(pt: PackedTrees, r: int) -> np.ndarray:
    """Columns row r attends to: itself and its ancestors (Fig 3), ascending."""
    return np.asarray(sorted([r] + ancestors(pt, r)), dtype=np.int64)


def dense_mask(pt: PackedTrees) -> np.ndarray:
    """[N, N] boolean visibility; small trees only."""
    N = pt.num_rows
    m = np.zeros((N, N), dtype=bool)
    for r in range(N):
        m[r, visible(pt, r)] = True
    return m


def positions(pt: PackedTrees) -> np.ndarray:
    """Semantic position of each row = number of strict ancestors (its depth).
    For trunk token j this is j; for y_{b,i} it is a_b + i.  Parents are
    packed before their children, so one pass in packed order counts them:
    depth(r) = depth(parent(r)) + 1, depth(root) = 0."""
    depth = np.zeros(pt.num_rows, dtype=np.int64)
    for r in range(pt.num_rows):
        p = int(pt.parent[r])
        if p >= 0:
            assert p < r, "parents are packed before their children"
            depth[r] = depth[p] + 1
    return depth


def prediction_rows(pt: PackedTrees) -> np.ndarray:
    """Readout row of prediction (b, i), i = 1..W, b-major: the row whose query
    predicts y_{b,i} is the parent of y_{b,i} in the tree, i.e. the anchor for
    i = 1 and y_{b,i-1} after that.  The terminal sample needs no row of its own."""
    out = []
    for b, rows in enumerate(pt.branch_rows):
        for i in range(1, pt.W + 1):
            if i == 1:
                out.append(int(pt.anchors_global[b]))
            else:
                out.append(rows[i - 2])
    return np.asarray(out, dtype=np.int64)


def row_fields(pt: PackedTrees, r: int):
    """Compact encoding of one row, read off its visible set vis(r):
    (pos, trunk_limit, branch_of, anc_bits) where
      pos          = |strict ancestors of r| (depth)
      trunk_limit  = largest tree-local trunk index in vis(r)
      branch_of    = global branch id of r (-1 on the trunk)
      anc_bits     = bit k-1 set iff y_{b,k} of r's own branch is in vis(r)
    """
    anc = ancestors(pt, r)
    vis = set(anc) | {r}
    trunk_cols = [int(pt.trunk_index[c]) for c in vis if pt.is_trunk[c]]
    b = int(pt.branch_of[r])
    acc = 0
    if b >= 0:
        for k, row in enumerate(pt.branch_rows[b], start=1):
            if row in vis:
                acc |= 1 << (k - 1)
    return len(anc), max(trunk_cols), b, acc


def compact_fields(pt: PackedTrees, rows=None):
    """Per-row compact encoding for ``rows`` (all rows by default), plus the
    prediction rows.  Values as in ``row_fields``."""
    if rows is None:
        rows = range(pt.num_rows)
    rows = list(rows)
    pos = np.zeros(len(rows), np.int64)
    tl = np.zeros(len(rows), np.int64)
    bof = np.zeros(len(rows), np.int64)
    bits = np.zeros(len(rows), np.uint64)
    for n, r in enumerate(rows):
        p, t, b, a = row_fields(pt, r)
        pos[n], tl[n], bof[n], bits[n] = p, t, b, np.uint64(a)
    return dict(pos=pos, trunk_limit=tl, branch_of=bof, anc_bits=bits,
                pred_rows=prediction_rows(pt))
