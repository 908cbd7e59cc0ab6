"""Short causal convolution along each packed row's own history (oracle; test
infrastructure only).

Source: "SpecOPD: Branch-Parallel On-Policy Distillation for Speculative
Decoding" as listed on thelatestinai.com, Fig 5: in the GDN branch path the
causal convolution follows branch ancestry, i.e. a branch token's convolution
window holds its own history, not its packed neighbours.

Readings where the pages are silent (plainest choice):
  * a depthwise causal 1-D convolution of width Kw over the row's history
    h = (x_0 .. x_{a_b}, y_{b,1} .. y_{b,i}) (the history of the tree-masked
    attention path; a trunk row's history is the trunk up to itself):
        out[r, c] = bias[c] + sum_{j=0}^{Kw-1} weight[c, j] * x[h_{-1-j}, c],
    weight[c, j] multiplying the token j steps back (j = 0: the row itself),
    positions before the start of the history reading zero;
  * an optional SiLU, act(u) = u / (1 + exp(-u)), applied after the sum (the
    gated delta rule's feature path convolves q, k and v, then applies SiLU).

Written from the definition in fp64, one row at a time.
"""
from __future__ import annotations

from typing import Optional, Sequence

import numpy as np

from . import tree as _tree


def history(pt: _tree.PackedTrees, r: int):
    """Packed rows of r's history, root first, r last."""
    return _tree.ancestors(pt, r)[::-1] + [r]


def tree_causal_conv(pt: _tree.PackedTrees, x: np.ndarray, weight: np.ndarray, bias: Optional[np.ndarray] = None,
                     silu: bool = False, rows: Optional[Sequence[int]] = None) -> np.ndarray:
    """x [N, C], weight [C, Kw], bias [C] or None -> [len(rows), C] (fp64; all
    rows by default)."""
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(weight, dtype=np.float64)
    N, C = x.shape
    Kw = w.shape[1]
    rows = list(range(N)) if rows is None else list(rows)
    out = np.zeros((len(rows), C))
    for n, r in enumerate(rows):
        hist = history(pt, r)
        acc = np.zeros(C) if bias is None else np.array(bias, dtype=np.float64)
        for j in range(Kw):
            if j < len(hist):
                acc = acc + w[:, j] * x[hist[-1 - j]]
        out[n] = acc / (1.0 + np.exp(-acc)) if silu else acc
    return out
