"""Pins for the oracle's gated delta rule over a proposal tree (CPU only).

What fixes the answers:
  * delta-rule memory: with beta = 1, alpha = 1 and orthonormal keys, writing
    (k_i, v_i) pairs stores them exactly, so the query k_j reads back v_j;
  * overwriting a key with v = 0 erases it whatever the decay alpha (the decay
    multiplies the whole update, I - beta k k^T included);
  * one step from the zero state: o = beta v (k . q); beta = 0 leaves S = 0;
  * pure decay: with beta = 0 after a write the output scales by the product
    of the alphas;
  * tree structure: a branch anchored at the last trunk token continues the
    trunk sequence; a branch never sees other branches or trunk tokens after
    its anchor; the C-token checkpoints equal the states of prefix runs;
  * the chunked (triangular-solve) formulation equals the sequential one for
    whole, ragged and single-token chunks and a non-zero start state.
"""
import numpy as np

from oracle import gdn as G
from oracle import tree as T


def _orthonormal(rng, n, d):
    q, _ = np.linalg.qr(rng.normal(size=(d, d)))
    return q[:, :n].T


def test_delta_rule_stores_and_recalls():
    rng = np.random.default_rng(0)
    dk, dv, n = 8, 5, 6
    keys = _orthonormal(rng, n, dk)
    vals = rng.normal(size=(n, dv))
    ones = np.ones(n)
    _, S = G.gdn_sequence(keys, keys, vals, ones, ones)
    for j in range(n):
        assert np.max(np.abs(S @ keys[j] - vals[j])) < 1e-12
    # the same key written twice keeps only the last value
    keys2 = np.vstack([keys[:1], keys[:1]])
    vals2 = rng.normal(size=(2, dv))
    _, S2 = G.gdn_sequence(keys2, keys2, vals2, np.ones(2), np.ones(2))
    assert np.max(np.abs(S2 @ keys[0] - vals2[1])) < 1e-12


def test_overwrite_with_zero_erases_under_decay():
    rng = np.random.default_rng(1)
    dk, dv = 6, 4
    k1 = _orthonormal(rng, 1, dk)[0]
    v1 = rng.normal(size=dv)
    k = np.vstack([k1, k1])
    v = np.vstack([v1, np.zeros(dv)])
    _, S = G.gdn_sequence(k, k, v, np.array([1.0, 0.5]), np.array([1.0, 1.0]))
    assert np.max(np.abs(S)) < 1e-13


def test_single_step_and_zero_write():
    rng = np.random.default_rng(2)
    q, k, v = rng.normal(size=(1, 5)), rng.normal(size=(1, 5)), rng.normal(size=(1, 3))
    o, _ = G.gdn_sequence(q, k, v, np.array([0.7]), np.array([0.3]))
    assert np.max(np.abs(o[0] - 0.3 * v[0] * float(k[0] @ q[0]))) < 1e-13
    o0, S0 = G.gdn_sequence(q, k, v, np.array([0.7]), np.array([0.0]))
    assert np.all(o0 == 0.0) and np.all(S0 == 0.0)


def test_pure_decay():
    rng = np.random.default_rng(3)
    dk, dv, L = 5, 3, 6
    q = np.tile(rng.normal(size=dk), (L, 1))
    k = rng.normal(size=(L, dk))
    v = rng.normal(size=(L, dv))
    alpha = rng.uniform(0.5, 1.0, size=L)
    beta = np.zeros(L)
    beta[0] = 0.8
    o, _ = G.gdn_sequence(q, k, v, alpha, beta)
    for t in range(1, L):
        assert np.max(np.abs(o[t] - o[0] * np.prod(alpha[1:t + 1]))) < 1e-13


def _tree_inputs(pt, H, dk, dv, seed):
    rng = np.random.default_rng(seed)
    N = pt.num_rows
    k = rng.normal(size=(N, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    return (rng.normal(size=(N, H, dk)), k, rng.normal(size=(N, H, dv)),
            rng.uniform(0.8, 1.0, size=(N, H)), rng.uniform(0.1, 0.9, size=(N, H)))


def test_branch_at_last_trunk_token_continues_the_trunk():
    Tn, W = 20, 4
    pt = T.pack([Tn], [5], [1], [Tn - 1], W, True)
    q, k, v, a, b = _tree_inputs(pt, 2, 6, 3, 4)
    out = G.gdn_tree(pt, q, k, v, a, b)
    for h in range(2):
        o, _ = G.gdn_sequence(q[:, h], k[:, h], v[:, h], a[:, h], b[:, h])   # rows are already in order
        assert np.max(np.abs(out[:, h] - o)) < 1e-12


def test_branch_isolation():
    Tn, W = 24, 3
    anchors = [10, 10, 17]
    pt = T.pack([Tn], [4], [3], anchors, W, True)
    q, k, v, a, b = _tree_inputs(pt, 1, 5, 4, 5)
    base = G.gdn_tree(pt, q, k, v, a, b)
    rows_b0 = [Tn, Tn + 1, Tn + 2]
    # change the sibling branch at the same anchor and every trunk token after the anchor
    v2 = v.copy()
    v2[Tn + 3:Tn + 6] += 1.0
    v2[11:Tn] += 1.0
    changed = G.gdn_tree(pt, q, k, v2, a, b)
    assert np.max(np.abs(changed[rows_b0] - base[rows_b0])) == 0.0
    assert np.max(np.abs(changed[Tn + 6:] - base[Tn + 6:])) > 0.0   # branch at 17 sees trunk 11..17


def test_checkpoints_are_prefix_states():
    rng = np.random.default_rng(6)
    Tn, H, dk, dv, C = 130, 2, 4, 3, 64
    q, k, v = rng.normal(size=(Tn, H, dk)), rng.normal(size=(Tn, H, dk)), rng.normal(size=(Tn, H, dv))
    a, b = rng.uniform(0.8, 1, size=(Tn, H)), rng.uniform(0, 1, size=(Tn, H))
    cp = G.checkpoint_states(q, k, v, a, b, Tn, C)
    assert cp.shape == (2, H, dv, dk)
    for j in (1, 2):
        for h in range(H):
            _, S = G.gdn_sequence(q[:C * j, h], k[:C * j, h], v[:C * j, h], a[:C * j, h], b[:C * j, h])
            assert np.max(np.abs(cp[j - 1, h] - S)) < 1e-12


def test_chunked_form_equals_the_sequential_recurrence():
    rng = np.random.default_rng(8)
    L, dk, dv = 70, 8, 5
    q, k, v = rng.normal(size=(L, dk)), rng.normal(size=(L, dk)), rng.normal(size=(L, dv))
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    alpha, beta = rng.uniform(0.7, 1.0, size=L), rng.uniform(0.0, 1.0, size=L)
    S0 = rng.normal(size=(dv, dk))
    o_ref, S_ref = G.gdn_sequence(q, k, v, alpha, beta, S0)
    for C in (1, 3, 16, 64, 100):                    # whole, ragged and single chunks
        o, S = G.gdn_sequence_chunked(q, k, v, alpha, beta, C, S0)
        assert np.max(np.abs(o - o_ref)) < 1e-10, C
        assert np.max(np.abs(S - S_ref)) < 1e-10, C
