"""Pins for the oracle's proposal-tree packing (CPU only).

What fixes the answers: the history definition h_{b,i} = (x_{<=a_b}, y_{b,<i})
(daiwk.github.io write-up, section "Equations"), the Fig 3 caption (each row sees
itself and its ancestors; siblings stay hidden), semantic positions a_b + i,
and the test list of the same write-up (future/sibling isolation, predecessor
readout, duplicate anchors, one-token branches).
"""
import numpy as np
import pytest

from oracle import tree as T


def history_visibility(trunk_len, prompt_len, num_branches, anchors, W, pack_terminal=True):
    """Visibility written straight from the history definition, without parents:
    trunk token j sees x_0..x_j of its tree; y_{b,i} sees x_0..x_{a_b} and y_{b,1..i}."""
    rpb = W if pack_terminal else W - 1
    N = sum(t + b * rpb for t, b in zip(trunk_len, num_branches))
    m = np.zeros((N, N), bool)
    base = 0
    a_off = 0
    for Tn, Bn in zip(trunk_len, num_branches):
        for j in range(Tn):
            m[base + j, base:base + j + 1] = True
        for b in range(Bn):
            a = anchors[a_off + b]
            start = base + Tn + b * rpb
            for i in range(1, rpb + 1):
                r = start + i - 1
                m[r, base:base + a + 1] = True
                m[r, start:start + i] = True
        base += Tn + Bn * rpb
        a_off += Bn
    return m


CASES = [
    # (trunk, prompt, branches), anchors, W, pack_terminal
    ([12], [3], [4], [3, 7, 11, 5], 3, True),
    ([12], [3], [4], [3, 7, 11, 5], 3, False),
    ([9], [2], [3], [4, 4, 4], 4, True),            # duplicate anchors
    ([10], [0], [5], [0, 9, 9, 1, 3], 1, True),     # one-token branches, P=0, a_b=T-1
    ([10], [4], [5], [4, 9, 6, 5, 8], 1, False),    # W=1 without terminal rows: no branch rows
    ([7, 5, 9], [2, 1, 3], [2, 0, 3], [6, 2, 3, 8, 4], 5, True),  # ragged multi-tree, a tree with no branches
]


@pytest.mark.parametrize("trunk,prompt,nb,anc,W,pt_flag", CASES)
def test_visibility_matches_history_definition(trunk, prompt, nb, anc, W, pt_flag):
    pt = T.pack(trunk, prompt, nb, anc, W, pt_flag)
    assert np.array_equal(T.dense_mask(pt), history_visibility(trunk, prompt, nb, anc, W, pt_flag))


@pytest.mark.parametrize("trunk,prompt,nb,anc,W,pt_flag", CASES)
def test_positions_are_semantic(trunk, prompt, nb, anc, W, pt_flag):
    pt = T.pack(trunk, prompt, nb, anc, W, pt_flag)
    pos = T.positions(pt)
    for r in range(pt.num_rows):
        if pt.is_trunk[r]:
            assert pos[r] == pt.trunk_index[r]
        else:
            b = pt.branch_of[r]
            a = pt.anchors_global[b] - pt.cu_rows[pt.tree_of[r]]
            assert pos[r] == a + pt.sample_index[r]


def test_semantic_positions_differ_from_packed_offsets():
    pt = T.pack([12], [3], [2], [4, 6], 3)
    pos = T.positions(pt)
    rows = pt.branch_rows[1]
    assert [int(pos[r]) for r in rows] == [7, 8, 9]
    assert rows == [15, 16, 17]


def test_sibling_and_future_isolation():
    pt = T.pack([12], [3], [3], [5, 5, 8], 4)
    m = T.dense_mask(pt)
    b0, b1, b2 = pt.branch_rows
    for r in b0:
        for c in b1 + b2:
            assert not m[r, c], "siblings (even at a duplicate anchor) are invisible"
    for i, r in enumerate(b0):
        for c in b0[i + 1:]:
            assert not m[r, c], "future samples are invisible"
    # trunk never sees branch rows; branch rows never see trunk beyond the anchor
    assert not m[:12, 12:].any()
    assert not m[b2[0], 9:12].any() and m[b2[0], :9].all()


def test_prediction_rows_are_predecessors_not_self():
    pt = T.pack([10], [2], [3], [2, 9, 5], 4)
    pred = T.prediction_rows(pt)
    for b, rows in enumerate(pt.branch_rows):
        for i in range(1, 5):
            r_pred = pred[b * 4 + i - 1]
            if i == 1:
                assert r_pred == pt.anchors_global[b]
            else:
                assert r_pred == rows[i - 2]
            # the readout row is the parent of y_{b,i}: own-row readout would leak the answer
            assert r_pred != rows[i - 1]
            assert pt.parent[rows[i - 1]] == r_pred


def test_terminal_rows_optional_without_changing_shared_rows():
    anc = [3, 7, 11, 5]
    a = T.pack([12], [3], [4], anc, 3, True)
    b = T.pack([12], [3], [4], anc, 3, False)
    ma, mb = T.dense_mask(a), T.dense_mask(b)
    # map rows of the terminal-free layout into the full layout
    idx = list(range(12))
    for rows in a.branch_rows:
        idx += rows[:-1]
    idx = np.asarray(idx)
    assert np.array_equal(ma[np.ix_(idx, idx)], mb)
    # readouts agree once re-indexed
    pa = T.prediction_rows(a)
    pb = T.prediction_rows(b)
    assert np.array_equal(pa, idx[pb])


def test_compact_fields_chain_encoding():
    pt = T.pack([7, 5], [1, 1], [2, 2], [3, 6, 1, 4], 5)
    f = T.compact_fields(pt)
    for r in range(pt.num_rows):
        if pt.is_trunk[r]:
            assert f["trunk_limit"][r] == pt.trunk_index[r] and f["anc_bits"][r] == 0
            assert f["branch_of"][r] == -1
        else:
            i = pt.sample_index[r]
            assert f["anc_bits"][r] == (1 << i) - 1
            b = pt.branch_of[r]
            assert f["trunk_limit"][r] == pt.anchors_global[b] - pt.cu_rows[pt.tree_of[r]]


def test_full_width_ancestor_bits():
    pt = T.pack([3], [0], [1], [2], 64)
    f = T.compact_fields(pt)
    assert int(f["anc_bits"][-1]) == (1 << 64) - 1


@pytest.mark.parametrize("anc", [[2], [12], [-1]])
def test_anchor_outside_reference_rejected(anc):
    with pytest.raises(T.TreeError):
        T.pack([12], [3], [1], anc, 2)


def test_bad_width_rejected():
    with pytest.raises(T.TreeError):
        T.pack([12], [3], [1], [5], 65)
    with pytest.raises(T.TreeError):
        T.pack([12], [3], [1], [5], 0)
