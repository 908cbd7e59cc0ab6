"""RoPE at semantic positions and tree-masked GQA attention (oracle; test
infrastructure only).

Definitions followed:
  * SpecOPD listing, Fig 3: one packed pass; each query row attends to itself
    and its ancestors, sharing trunk keys/values.
  * daiwk.github.io write-up, section "Equations": semantic positions a_b + i
    (not packed offsets) for branch tokens.
  * same write-up, section "Inputs and code mapping": packed scoring equals each
    branch's independent causal scoring (the second formulation below).

Readings where the pages are silent (plainest choice): rotate-half RoPE with
frequency theta^(-2k/d) pairing element k with k + d/2; softmax scale 1/sqrt(d)
with no soft-cap, window or bias; query head h reads KV head h // (Hq/Hkv).

Everything runs in fp64 on exact upcasts of the stored inputs.
"""
from __future__ import annotations

from typing import Iterable, Optional

import numpy as np

from . import tree as _tree


def rope(x: np.ndarray, pos: np.ndarray, theta: float) -> np.ndarray:
    """Rotate-half rotary embedding of x [N, H, d] at integer positions pos [N]."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    half = d // 2
    inv_freq = theta ** (-2.0 * np.arange(half, dtype=np.float64) / d)
    ang = np.asarray(pos, dtype=np.float64)[:, None] * inv_freq[None, :]
    cos = np.cos(ang)[:, None, :]
    sin = np.sin(ang)[:, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * cos - x2 * sin, x2 * cos + x1 * sin], axis=-1)


def _softmax_attend(qh: np.ndarray, kc: np.ndarray, vc: np.ndarray, scale: float) -> np.ndarray:
    """One query vector against the listed keys/values: softmax(q.k * scale) . v."""
    s = (kc @ qh) * scale
    s = s - s.max()
    w = np.exp(s)
    w /= w.sum()
    return w @ vc


def tree_attention(pt: _tree.PackedTrees, q: np.ndarray, k: np.ndarray, v: np.ndarray,
                   theta: float, scale: Optional[float] = None,
                   rows: Optional[Iterable[int]] = None) -> np.ndarray:
    """O[r, h] = softmax over c in vis(r) of (RoPE(q_r) . RoPE(k_c)) * scale, applied to v_c.

    q [N, Hq, d], k/v [N, Hkv, d] (fp64 or exactly upcast), RoPE at the
    semantic positions (depths) of the packed rows.  Returns [len(rows), Hq, d]
    (all rows by default).
    """
    N, Hq, d = q.shape
    Hkv = k.shape[1]
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    grp = Hq // Hkv
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    pos = _tree.positions(pt)
    rows = list(range(N)) if rows is None else list(rows)
    qr = rope(np.asarray(q)[rows], pos[rows], theta)
    kr = rope(k, pos, theta)
    vv = np.asarray(v, dtype=np.float64)
    out = np.zeros((len(rows), Hq, d), dtype=np.float64)
    for n, r in enumerate(rows):
        cols = _tree.visible(pt, r)
        for h in range(Hq):
            g = h // grp
            out[n, h] = _softmax_attend(qr[n, h], kr[cols, g], vv[cols, g], scale)
    return out


def branch_causal_attention(pt: _tree.PackedTrees, q: np.ndarray, k: np.ndarray, v: np.ndarray,
                            theta: float, scale: Optional[float] = None) -> np.ndarray:
    """Second formulation, for the self-check: every row is scored by plain
    causal attention over its own sequence, with RoPE at the natural positions
    0..L-1 of that sequence.

    * trunk rows of a tree: causal attention over the trunk x_0..x_{T-1};
    * rows of branch b: causal attention over (x_0..x_{a_b}, y_{b,1}, y_{b,2}, ...),
      the sequence a drafter history h_{b,i} is made of.

    Uses torch's CPU scaled_dot_product_attention(is_causal=True) in fp64, a
    library routine independent of ``tree_attention``.
    """
    import torch
    import torch.nn.functional as F

    N, Hq, d = q.shape
    Hkv = k.shape[1]
    grp = Hq // Hkv
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    out = np.zeros((N, Hq, d), dtype=np.float64)

    def causal(seq_rows: np.ndarray) -> np.ndarray:
        L = seq_rows.shape[0]
        nat = np.arange(L)
        qs = rope(q[seq_rows], nat, theta)            # [L, Hq, d]
        ks = rope(k[seq_rows], nat, theta)            # [L, Hkv, d]
        vs = np.asarray(v[seq_rows], dtype=np.float64)
        ks = np.repeat(ks, grp, axis=1)
        vs = np.repeat(vs, grp, axis=1)
        tq = torch.from_numpy(np.ascontiguousarray(qs.transpose(1, 0, 2)))
        tk = torch.from_numpy(np.ascontiguousarray(ks.transpose(1, 0, 2)))
        tv = torch.from_numpy(np.ascontiguousarray(vs.transpose(1, 0, 2)))
        o = F.scaled_dot_product_attention(tq, tk, tv, is_causal=True, scale=scale)
        return o.numpy().transpose(1, 0, 2)

    ntrees = pt.cu_rows.shape[0] - 1
    for t in range(ntrees):
        trunk = np.nonzero((pt.tree_of == t) & pt.is_trunk)[0]
        out[trunk] = causal(trunk)
    for b, rows in enumerate(pt.branch_rows):
        if not rows:
            continue
        a = int(pt.anchors_global[b])
        t = int(pt.tree_of[a])
        base = int(pt.cu_rows[t])
        seq = np.concatenate([np.arange(base, a + 1), np.asarray(rows, np.int64)])
        o = causal(seq)
        out[rows] = o[-len(rows):]
    return out
