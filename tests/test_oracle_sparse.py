"""Pins for the oracle's sparse attention with branch-consistent indexer groups
(CPU only).

What fixes the answers:
  * with k at least the number of complete groups every group is selected,
    so the result is the full tree attention of attention.py (itself pinned to
    per-branch causal attention);
  * a branch row equals the same row in a tree made of that branch's own
    sequence (the trunk cut at the anchor), so nothing leaks across branches;
  * a constructed indexer that makes one group win selects exactly that
    group's members plus the causal tail;
  * the group a branch token completes is keyed by that branch's own token:
    two branches at one anchor select it or not according to their own key;
  * the causal tail (the row's incomplete group) is attended whatever the
    indexer says.
"""
import numpy as np

from oracle import attention as A
from oracle import sparse as SP
from oracle import tree as T


def _inputs(N, Hq, Hkv, d, di, seed):
    rng = np.random.default_rng(seed)
    return (rng.normal(size=(N, Hq, d)), rng.normal(size=(N, Hkv, d)), rng.normal(size=(N, Hkv, d)),
            rng.normal(size=(N, Hkv, di)), rng.normal(size=(N, Hkv, di)))


def test_large_k_is_full_tree_attention():
    pt = T.pack([30, 17], [4, 2], [3, 2], [10, 20, 29, 5, 16], 4, True)
    q, k, v, qi, ki = _inputs(pt.num_rows, 4, 2, 8, 4, 0)
    for g in (1, 3, 4):
        got = SP.sparse_tree_attention(pt, q, k, v, qi, ki, g, 1000, 1e4)
        ref = A.tree_attention(pt, q, k, v, 1e4)
        assert np.max(np.abs(got - ref)) < 1e-12


def test_branch_row_equals_its_own_sequence():
    Tn, W, g, topk = 26, 5, 3, 2
    anchors = [11, 11, 20]
    pt = T.pack([Tn], [3], [3], anchors, W, True)
    q, k, v, qi, ki = _inputs(pt.num_rows, 2, 1, 8, 4, 1)
    got = SP.sparse_tree_attention(pt, q, k, v, qi, ki, g, topk, 1e4)
    for b, a in enumerate(anchors):
        # one tree: the trunk through the anchor, the branch anchored at its end
        sub = T.pack([a + 1], [3], [1], [a], W, True)
        idx = list(range(a + 1)) + list(range(Tn + b * W, Tn + (b + 1) * W))
        ref = SP.sparse_tree_attention(sub, q[idx], k[idx], v[idx], qi[idx], ki[idx], g, topk, 1e4)
        assert np.max(np.abs(got[Tn + b * W:Tn + (b + 1) * W] - ref[a + 1:])) < 1e-12


def test_constructed_selection():
    Tn, g = 9, 2
    pt = T.pack([Tn], [0], [0], [], 1, True)
    di = 3
    q, k, v, _, _ = _inputs(Tn, 1, 1, 4, di, 2)
    qi = np.zeros((Tn, 1, di))
    ki = np.zeros((Tn, 1, di))
    qi[6, 0] = [1.0, 0.0, 0.0]
    ki[2, 0] = ki[3, 0] = [5.0, 0.0, 0.0]   # group 1 (positions 2, 3) scores 5; groups 0 and 2 score 0
    cols = SP.selected_columns(pt, 6, qi, ki, g, 1, 0)
    assert cols == [2, 3, 6]                # group 1 plus the tail (position 6, its group incomplete)
    out = SP.sparse_tree_attention(pt, q, k, v, qi, ki, g, 1, 1e4, rows=[6])
    pos = T.positions(pt)
    qr, kr = A.rope(q, pos, 1e4), A.rope(k, pos, 1e4)
    s = np.array([qr[6, 0] @ kr[c, 0] for c in cols]) / 2.0
    w = np.exp(s - s.max())
    w /= w.sum()
    assert np.max(np.abs(out[0, 0] - w @ v[cols, 0])) < 1e-12
    # ties go to the earlier group
    assert SP.selected_columns(pt, 7, np.zeros((Tn, 1, di)), np.zeros((Tn, 1, di)), g, 1, 0) == [0, 1]


def test_branch_specific_boundary_group():
    Tn, W, g = 12, 2, 4
    a = 6                                     # positions 4, 5, 6 form an incomplete trunk group
    pt = T.pack([Tn], [0], [2], [a, a], W, True)
    N, di = pt.num_rows, 2
    qi = np.zeros((N, 1, di))
    ki = np.zeros((N, 1, di))
    y0, y1 = Tn, Tn + W                       # the first token of each branch (position 7)
    qi[y0, 0] = qi[y1, 0] = [1.0, 0.0]
    ki[y0, 0] = [10.0, 0.0]                   # branch 0's token lifts the completed group's mean key
    ki[y1, 0] = [-10.0, 0.0]                  # branch 1's token sinks it
    ki[0:4, 0] = [0.5, 0.0]                   # trunk group 0 scores 0.5
    c0 = SP.selected_columns(pt, y0, qi, ki, g, 1, 0)
    c1 = SP.selected_columns(pt, y1, qi, ki, g, 1, 0)
    assert c0 == [4, 5, 6, y0]                # the branch-keyed group (score 2.5) wins; no tail
    assert c1 == [0, 1, 2, 3]                 # its own group scores -2.5: trunk group 0 wins


def test_tail_bypasses_top_k():
    pt = T.pack([10], [0], [0], [], 1, True)
    qi = np.zeros((10, 1, 2))
    ki = np.zeros((10, 1, 2))
    ki[0:3, 0] = [1.0, 1.0]
    qi[:, 0] = [1.0, 1.0]
    for r in range(10):
        cols = SP.selected_columns(pt, r, qi, ki, 3, 1, 0)
        tail = list(range((r + 1) // 3 * 3, r + 1))
        assert cols[len(cols) - len(tail):] == tail
        assert r in cols or (r + 1) % 3 == 0


def test_exact_ties_pick_the_earliest_groups():
    pt = T.pack([33], [0], [1], [20], 4, True)
    N = pt.num_rows
    zeros = np.zeros((N, 1, 8))
    for r in (10, 32, 33, 36):
        cols = SP.selected_columns(pt, r, zeros, zeros, 4, 2, 0)
        hist = SP.history(pt, r)
        p = len(hist) - 1
        nc = (p + 1) // 4
        expect = hist[:min(nc, 2) * 4] + hist[nc * 4:]
        assert cols == expect, r


def test_top_groups_order_and_count():
    s = np.array([0.5, 2.0, -1.0, 2.0, 0.7])
    assert SP.top_groups(s, 2) == [1, 3]          # the two best, ascending
    assert SP.top_groups(s, 3) == [1, 3, 4]
    assert SP.top_groups(np.array([1.0, 1.0, 1.0]), 2) == [0, 1]   # ties to the earlier group
    assert SP.top_groups(s, 9) == [0, 1, 2, 3, 4]  # k above the count: every group


def test_group_scores_are_query_dot_member_mean():
    """Brute force for one branch row: each complete group's score is the
    indexer query dotted with the mean of its members' keys, the members
    being the row's own history (trunk through the anchor, then its branch)."""
    pt = T.pack([10], [2], [2], [5, 8], 4, True)
    rng = np.random.default_rng(3)
    qi = rng.standard_normal((pt.num_rows, 1, 6))
    ki = rng.standard_normal((pt.num_rows, 1, 6))
    r = 10 + 4 + 2            # y_{1,3} of the branch at anchor 8: history x_0..x_8, y_{1,1}, y_{1,2}, y_{1,3}
    hist = list(range(0, 9)) + [14, 15, 16]
    assert SP.history(pt, r) == hist
    got = SP.group_scores(pt, r, qi, ki, 3, 0)
    want = [sum(qi[r, 0, e] * sum(ki[hist[m * 3 + j], 0, e] for j in range(3)) / 3 for e in range(6))
            for m in range(4)]
    assert np.allclose(got, want, rtol=0, atol=1e-12)
