"""Full-vocabulary overlap, E2E-TV loss and its gradient (oracle; test
infrastructure only).

Definitions followed (daiwk.github.io write-up of SpecOPD):
  * section "Equations": alpha_{b,i} = sum_v min(q(v|h_{b,i}), p(v|h_{b,i}));
    L = 1 - (1/(B W)) sum_b sum_{j=1..W} prod_{i<=j} alpha_{b,i};
    samples and teacher are fixed during differentiation; teacher mass outside
    the draft support is kept, never renormalised away.
  * section "Inputs and code mapping": inactive draft-support entries may hold
    NaN padding; the whole teacher vocabulary must stay finite; fp16/bf16
    probability work is promoted (here: everything is fp64).
  * section "Checks, negative controls, and limits": the worked example
    q = [.5, .5, 0] against p = [.4, .4, .2] gives loss .2.

Readings where the pages are silent (plainest choice):
  * a draft logit that is NaN or -inf marks an inactive entry (q = 0 there,
    gradient 0); +inf is an error; any non-finite teacher logit is an error;
    a row with no active entry has q = 0 everywhere and alpha = 0.
  * logits are used at temperature 1.
  * the gradient of min at an exact tie q(v) = p(v) takes the teacher branch
    (the draft side counts only where q(v) < p(v) strictly).
  * one batch of several trees is one loss, normalised by the total number of
    predictions sum_b W.
"""
from __future__ import annotations

import numpy as np


class NonFiniteError(ValueError):
    pass


def draft_probs(z: np.ndarray):
    """Draft distribution q over the active support of each row (softmax of the
    active logits; inactive entries get 0).  Returns (q, active, log_q)."""
    z = np.asarray(z, dtype=np.float64)
    if np.any(np.isposinf(z)):
        raise NonFiniteError("draft logit +inf")
    active = np.isfinite(z)
    zz = np.where(active, z, -np.inf)
    m = zz.max(axis=-1, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    e = np.where(active, np.exp(zz - m), 0.0)
    s = e.sum(axis=-1, keepdims=True)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.where(s > 0, e / np.where(s > 0, s, 1.0), 0.0)
        log_q = np.where(active & (s > 0), zz - m - np.log(np.where(s > 0, s, 1.0)), -np.inf)
    return q, active, log_q


def teacher_probs(t: np.ndarray):
    """Teacher distribution p = softmax(t) over the full vocabulary (never
    restricted to the draft support).  Returns (p, log_p)."""
    t = np.asarray(t, dtype=np.float64)
    if not np.all(np.isfinite(t)):
        raise NonFiniteError("teacher logits must be finite")
    m = t.max(axis=-1, keepdims=True)
    e = np.exp(t - m)
    s = e.sum(axis=-1, keepdims=True)
    return e / s, t - m - np.log(s)


def overlap(z: np.ndarray, t: np.ndarray) -> np.ndarray:
    """alpha[row] = sum_v min(q_v, p_v)."""
    q, _, _ = draft_probs(z)
    p, _ = teacher_probs(t)
    return np.minimum(q, p).sum(axis=-1)


def e2e_tv_loss(alpha: np.ndarray, W: int, count: int = None) -> float:
    """L = 1 - (1/count) sum_b sum_j prod_{i<=j} alpha_{b,i}; alpha is b-major
    [sum B * W]; count defaults to the number of predictions.  An empty batch
    has no predictions and no loss: 0 is returned."""
    a = np.asarray(alpha, dtype=np.float64).reshape(-1, W)
    if count is None:
        count = a.size
    if count == 0:
        return 0.0
    total = 0.0
    for b in range(a.shape[0]):
        for j in range(W):
            total += float(np.prod(a[b, :j + 1]))
    return 1.0 - total / count


def e2e_tv_grad_alpha(alpha: np.ndarray, W: int, count: int = None) -> np.ndarray:
    """dL/dalpha_{b,i} = -(1/count) sum_{j>=i} prod_{k<=j, k!=i} alpha_{b,k}
    (product rule applied to every prefix product containing alpha_{b,i})."""
    a = np.asarray(alpha, dtype=np.float64).reshape(-1, W)
    if count is None:
        count = a.size
    g = np.zeros_like(a)
    if count == 0:
        return g.reshape(-1)
    for b in range(a.shape[0]):
        for i in range(W):
            acc = 0.0
            for j in range(i, W):
                acc += float(np.prod(np.delete(a[b, :j + 1], i)))
            g[b, i] = -acc / count
    return g.reshape(-1)


def overlap_grad_draft(z: np.ndarray, t: np.ndarray) -> np.ndarray:
    """d alpha / d z_u for every row: the derivative of sum_v min(q_v, p_v) with
    p fixed.  Where q_v < p_v the term is q_v, whose derivative through the
    softmax is q_v (delta_vu - q_u); elsewhere it is the constant p_v.  Summing:
    q_u ([q_u < p_u] - sum_v q_v [q_v < p_v]).  Inactive entries get 0."""
    q, active, log_q = draft_probs(z)
    _, log_p = teacher_probs(t)
    m = (log_q < log_p) & active
    q_less = (q * m).sum(axis=-1, keepdims=True)
    return np.where(active, q * (m.astype(np.float64) - q_less), 0.0)


def e2e_tv_grad_draft(z: np.ndarray, t: np.ndarray, W: int, count: int = None) -> np.ndarray:
    """dL/dz = (dL/dalpha)_row * (d alpha/d z)_row, teacher and samples fixed."""
    alpha = overlap(z, t)
    ga = e2e_tv_grad_alpha(alpha, W, count)
    return ga[:, None] * overlap_grad_draft(z, t)


def loss_from_logits(z: np.ndarray, t: np.ndarray, W: int, count: int = None) -> float:
    """Forward of the whole objective from logits (used by the finite-difference pin)."""
    return e2e_tv_loss(overlap(z, t), W, count)
