"""Gated DeltaNet (GDN) linear attention over a proposal tree: every packed row
reads the recurrent state of its own history (oracle; test infrastructure only).

Source: "SpecOPD: Branch-Parallel On-Policy Distillation for Speculative
Decoding" as listed on thelatestinai.com, Fig 5: a shared trunk pass caches an
fp32 GDN state at every C = 64 boundary; each branch loads the checkpoint at or
before its anchor, replays the cached trunk features up to the anchor, then
updates the state over its own tokens and reads it with each token's query;
checkpoints stay immutable.

Readings where the pages are silent (plainest choice):
  * the recurrence is the gated delta rule, per head, with the state
    S in R^{d_v x d_k} starting at zero:
        S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
        o_t = S_t q_t,
    alpha_t in (0, 1] the decay gate, beta_t in [0, 1] the write strength;
  * q, k, v, alpha, beta are per-token features already produced upstream
    (projections, the short causal convolution over the branch's ancestry,
    key normalisation); this path consumes them as given;
  * a branch's history is the trunk through its anchor a_b followed by its own
    earlier tokens, the history of the tree-masked attention path.

This module writes the definition out: one sequential pass per history, in
fp64, with no chunking and no checkpoints.  `checkpoint_states` returns the
trunk states at the C-token boundaries the GPU path caches, from the same
sequential pass.
"""
from __future__ import annotations

import numpy as np

from . import tree as _tree


def gdn_sequence(q: np.ndarray, k: np.ndarray, v: np.ndarray, alpha: np.ndarray, beta: np.ndarray,
                 state: np.ndarray = None):
    """One head over one sequence.  q, k [L, dk], v [L, dv], alpha, beta [L].
    Returns (o [L, dv], final state [dv, dk]); `state` is the starting state
    (zero if None)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    L, dk = k.shape
    dv = v.shape[1]
    S = np.zeros((dv, dk)) if state is None else np.array(state, dtype=np.float64)
    o = np.zeros((L, dv))
    eye = np.eye(dk)
    for t in range(L):
        kt = k[t][:, None]
        S = float(alpha[t]) * S @ (eye - float(beta[t]) * (kt @ kt.T)) + float(beta[t]) * (v[t][:, None] @ kt.T)
        o[t] = S @ q[t]
    return o, S


def gdn_tree(pt: _tree.PackedTrees, q: np.ndarray, k: np.ndarray, v: np.ndarray, alpha: np.ndarray,
             beta: np.ndarray) -> np.ndarray:
    """All packed rows.  q, k [N, H, dk], v [N, H, dv], alpha, beta [N, H].
    Row r's output is the recurrence over its history (its ancestors in packed
    order, then itself), read with its own query."""
    N, H = q.shape[0], q.shape[1]
    out = np.zeros((N, H, v.shape[2]))
    for r in range(N):
        hist = _tree.ancestors(pt, r)[::-1] + [r]   # root first
        for h in range(H):
            o, _ = gdn_sequence(q[hist, h], k[hist, h], v[hist, h], alpha[hist, h], beta[hist, h])
            out[r, h] = o[-1]
    return out


def checkpoint_states(q: np.ndarray, k: np.ndarray, v: np.ndarray, alpha: np.ndarray, beta: np.ndarray,
                      T: int, C: int = 64) -> np.ndarray:
    """States after trunk tokens C j - 1 for j = 1 .. T // C of one tree's trunk
    (rows 0 .. T-1 of q, k, v, alpha, beta): [T // C, H, dv, dk]."""
    H = q.shape[1]
    out = np.zeros((T // C, H, v.shape[2], k.shape[2]))
    for h in range(H):
        S = None
        for j in range(T // C):
            sl = slice(j * C, (j + 1) * C)
            _, S = gdn_sequence(q[sl, h], k[sl, h], v[sl, h], alpha[sl, h], beta[sl, h], S)
            out[j, h] = S
    return out


def gdn_sequence_chunked(q: np.ndarray, k: np.ndarray, v: np.ndarray, alpha: np.ndarray, beta: np.ndarray,
                         C: int, state: np.ndarray = None):
    """The same recurrence as gdn_sequence, C tokens at a time (a second
    formulation, checked against the sequential one; it is the chunked form a
    tensor-core trunk pass follows).

    Within a chunk with start state S0, cumulative decays g_t = prod_{i<=t}
    alpha_i and update vectors u_t (S_t = alpha_t S_{t-1} + u_t k_t^T), the
    delta rule gives
        u_t + beta_t sum_{i<t} (g_t / g_i) (k_t . k_i) u_i = beta_t (v_t - g_t S0 k_t),
    a unit lower-triangular system (I + A) U = diag(beta) (V - diag(g) K S0^T);
    then
        O   = diag(g) Q S0^T + (L o (Q K^T)) U,   L_ti = g_t / g_i for i <= t,
        S_C = g_C S0 + (diag(g_C / g) U)^T K.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    alpha = np.asarray(alpha, dtype=np.float64)
    beta = np.asarray(beta, dtype=np.float64)
    L, dk = k.shape
    dv = v.shape[1]
    S = np.zeros((dv, dk)) if state is None else np.array(state, dtype=np.float64)
    o = np.zeros((L, dv))
    for c0 in range(0, L, C):
        sl = slice(c0, min(L, c0 + C))
        qc, kc, vc, bc = q[sl], k[sl], v[sl], beta[sl]
        lg = np.cumsum(np.log(alpha[sl]))              # log g_t
        n = kc.shape[0]
        ratio = np.exp(lg[:, None] - lg[None, :])      # g_t / g_i
        A = np.tril(bc[:, None] * ratio * (kc @ kc.T), -1)
        rhs = bc[:, None] * (vc - np.exp(lg)[:, None] * (kc @ S.T))
        U = np.zeros((n, dv))
        for t in range(n):                             # forward substitution, unit diagonal
            U[t] = rhs[t] - A[t, :t] @ U[:t]
        Lmask = np.tril(ratio)
        o[sl] = np.exp(lg)[:, None] * (qc @ S.T) + (Lmask * (qc @ kc.T)) @ U
        S = np.exp(lg[-1]) * S + (np.exp(lg[-1] - lg)[:, None] * U).T @ kc
    return o, S
