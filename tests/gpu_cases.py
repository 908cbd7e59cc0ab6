"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI
on a synthetic case and compute the matching oracle values."""
from __future__ import annotations

import numpy as np
import torch

from oracle import attention as OA
from oracle import overlap as OO
from oracle import tree as OT
from synthetic import Case, to_f64


def torch_dtype(case: Case):
    return torch.bfloat16 if case.dtype == "bf16" else torch.float32


def step_for(case: Case, with_grad: bool = True):
    from tree_attention_masked_b200.build import build
    build()
    from tree_attention_masked_b200.scoring import ScoringStep
    st = ScoringStep(case.trunk_len, case.prompt_len, case.num_branches, case.W, case.Hq, case.Hkv, case.d,
                     torch_dtype(case), case.vocab if case.teacher is not None else 1,
                     pack_terminal=case.pack_terminal, theta=case.theta,
                     with_grad=with_grad)
    st.load(case)
    return st


def to_np(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy().astype(np.float64)
    return t.cpu().numpy()


def packed(case: Case) -> OT.PackedTrees:
    return OT.pack(case.trunk_len, case.prompt_len, case.num_branches, case.anchors, case.W, case.pack_terminal)


def expected_tile_meta(pt: OT.PackedTrees, fields) -> np.ndarray:
    """Per-tile column ranges, computed from the oracle's per-row fields."""
    rows = []
    ntrees = pt.cu_rows.shape[0] - 1
    for t in range(ntrees):
        base, end = int(pt.cu_rows[t]), int(pt.cu_rows[t + 1])
        for r0 in range(base, end, 128):
            r1 = min(end, r0 + 128)
            lims = [base + int(fields["trunk_limit"][r]) + 1 for r in range(r0, r1)]
            br = [r for r in range(r0, r1) if fields["branch_of"][r] >= 0]
            if br:
                lo = min(r - int(pt.sample_index[r]) + 1 for r in br)
                hi = max(br) + 1
            else:
                lo = hi = 0
            rows.append([r0, r1, base, max(lims), min(lims), lo, hi, 0])
    return np.asarray(rows, dtype=np.int64).reshape(-1, 8)


def oracle_attention_rows(case: Case, pt: OT.PackedTrees, rows) -> np.ndarray:
    q = to_f64(case.q, case.dtype)
    k = to_f64(case.k, case.dtype)
    v = to_f64(case.v, case.dtype)
    return OA.tree_attention(pt, q, k, v, theta=case.theta, rows=rows)


def rel_l2(a: np.ndarray, b: np.ndarray) -> float:
    return float(np.linalg.norm((a - b).ravel()) / max(np.linalg.norm(b.ravel()), 1e-300))


def oracle_overlap(case: Case, rows=None):
    """alpha for the given prediction rows (all by default)."""
    z = to_f64(case.draft if rows is None else case.draft[rows], case.dtype)
    t = to_f64(case.teacher if rows is None else case.teacher[rows], case.dtype)
    return OO.overlap(z, t)


def oracle_overlap_chunked(case: Case, chunk: int = 64) -> np.ndarray:
    R = case.draft.shape[0]
    out = np.empty(R, dtype=np.float64)
    for r0 in range(0, R, chunk):
        out[r0:r0 + chunk] = oracle_overlap(case, np.arange(r0, min(R, r0 + chunk)))
    return out


def oracle_branch_grad(case: Case, b: int, count: int) -> np.ndarray:
    W = case.W
    rows = np.arange(b * W, (b + 1) * W)
    z = to_f64(case.draft[rows], case.dtype)
    t = to_f64(case.teacher[rows], case.dtype)
    return OO.e2e_tv_grad_draft(z, t, W, count=count)
