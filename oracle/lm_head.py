"""Prediction logits from hidden states and a head, and the overlap and E2E-TV
statistics taken from them (oracle; test infrastructure only).

Definitions followed (daiwk.github.io write-up of SpecOPD):
  * section "Inputs and code mapping": prediction_logits reads supplied hidden
    states and a supplied head (not a teacher checkpoint); e2e_tv_loss then
    consumes the same-history aligned logits of draft and teacher.
  * section "Equations": alpha, L and the fixed teacher, as in overlap.py.

Reading where the pages are silent (plainest choice): the logits of a row are
the products of its hidden state with every row of the head, logits = h W^T
(W holds one row of hidden size per vocabulary entry), with no bias, no
normalisation and temperature 1.  Draft and teacher each have their own
hidden states and head; the vocabulary is shared and every entry is active.

Every quantity is fp64 from the (bf16-exact) inputs; the logits are formed
with one matrix product (a library primitive) and then handed to the
definitions in overlap.py unchanged.
"""
from __future__ import annotations

import numpy as np

from . import overlap as _ov


def prediction_logits(h: np.ndarray, head: np.ndarray) -> np.ndarray:
    """logits[r, v] = sum_k h[r, k] * head[v, k] (fp64)."""
    h = np.asarray(h, dtype=np.float64)
    head = np.asarray(head, dtype=np.float64)
    if h.ndim != 2 or head.ndim != 2 or h.shape[1] != head.shape[1]:
        raise ValueError("h [rows, H] and head [V, H] must share H")
    return h @ head.T


def row_statistics(z: np.ndarray, t: np.ndarray) -> dict:
    """Per-row natural-log normalisers of draft and teacher, alpha and
    q_less = sum_v q_v [q_v < p_v] (strict, compared in the log domain)."""
    q, active, log_q = _ov.draft_probs(z)
    p, log_p = _ov.teacher_probs(t)
    zz = np.where(active, np.asarray(z, dtype=np.float64), -np.inf)
    mz = zz.max(axis=-1)
    lse_draft = mz + np.log(np.exp(zz - mz[:, None]).sum(axis=-1))
    tt = np.asarray(t, dtype=np.float64)
    mt = tt.max(axis=-1)
    lse_teacher = mt + np.log(np.exp(tt - mt[:, None]).sum(axis=-1))
    less = (log_q < log_p) & active
    return {
        "alpha": np.minimum(q, p).sum(axis=-1),
        "q_less": (q * less).sum(axis=-1),
        "lse_draft": lse_draft,
        "lse_teacher": lse_teacher,
    }


def lm_head_overlap(h_draft: np.ndarray, head_draft: np.ndarray, h_teacher: np.ndarray,
                    head_teacher: np.ndarray, W: int, count: int = None) -> dict:
    """alpha, q_less, both normalisers, L and dL/dalpha for prediction rows
    given as hidden states (b-major rows, W per branch)."""
    z = prediction_logits(h_draft, head_draft)
    t = prediction_logits(h_teacher, head_teacher)
    out = row_statistics(z, t)
    out["loss"] = _ov.e2e_tv_loss(out["alpha"], W, count)
    out["grad_alpha"] = _ov.e2e_tv_grad_alpha(out["alpha"], W, count)
    return out
