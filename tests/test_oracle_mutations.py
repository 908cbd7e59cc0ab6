"""Planted mistakes: each plausible slip in the oracle must break one of its pins.

Each test swaps one oracle function for a subtly wrong variant (on the CPU,
inside the test only) and checks that the matching pin from the other test
files now fails.  This shows the pins constrain the oracle rather than restate it.
"""
import json
import os

import numpy as np

from oracle import attention as A
from oracle import overlap as O
from oracle import tree as T

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "worked_example.json")))


def _worked_loss(overlap_fn):
    q = np.asarray(GOLD["draft_q"])
    p = np.asarray(GOLD["teacher_p"])
    with np.errstate(divide="ignore"):
        z = np.log(q)[None, :]
    return O.e2e_tv_loss(overlap_fn(z, np.log(p)[None, :]), 1)


def test_renormalised_teacher_breaks_worked_example():
    def bad_overlap(z, t):
        q, active, _ = O.draft_probs(z)
        p, _ = O.teacher_probs(t)
        p = np.where(active, p, 0.0)
        p = p / p.sum(axis=-1, keepdims=True)
        return np.minimum(q, p).sum(axis=-1)
    assert abs(_worked_loss(O.overlap) - GOLD["loss"]) < 1e-15
    assert abs(_worked_loss(bad_overlap) - GOLD["loss"]) > 0.1


def test_max_instead_of_min_breaks_worked_example():
    def bad_overlap(z, t):
        q, _, _ = O.draft_probs(z)
        p, _ = O.teacher_probs(t)
        return np.maximum(q, p).sum(axis=-1)
    assert abs(_worked_loss(bad_overlap) - GOLD["loss"]) > 0.1


def _fd_max_error(grad_fn):
    rng = np.random.default_rng(5)
    W, V = 3, 6
    t = rng.normal(0, 2, (2 * W, V))
    z = t + rng.normal(0, 1, (2 * W, V))
    g = grad_fn(z, t, W)
    h = 1e-6
    err = 0.0
    for r in range(z.shape[0]):
        for u in range(V):
            zp, zm = z.copy(), z.copy()
            zp[r, u] += h
            zm[r, u] -= h
            fd = (O.loss_from_logits(zp, t, W) - O.loss_from_logits(zm, t, W)) / (2 * h)
            err = max(err, abs(fd - g[r, u]))
    return err


def test_gradient_slips_break_finite_differences():
    assert _fd_max_error(O.e2e_tv_grad_draft) < 1e-8

    def dropped_term(z, t, W):
        q, active, log_q = O.draft_probs(z)
        _, log_p = O.teacher_probs(t)
        m = (log_q < log_p) & active
        ga = O.e2e_tv_grad_alpha(O.overlap(z, t), W)
        return ga[:, None] * q * m

    def wrong_sign(z, t, W):
        return -O.e2e_tv_grad_draft(z, t, W)

    def wrong_row(z, t, W):
        g = O.e2e_tv_grad_draft(z, t, W)
        return np.roll(g, 1, axis=0)

    for bad in (dropped_term, wrong_sign, wrong_row):
        assert _fd_max_error(bad) > 1e-4


def test_prefix_off_by_one_breaks_enumeration_pin():
    from tests.test_oracle_overlap import expected_prefix_by_enumeration
    rng = np.random.default_rng(2)
    W = 4
    a = rng.uniform(0, 1, W)

    def bad_loss(alpha, W):
        alpha = np.asarray(alpha).reshape(-1, W)
        tot = sum(float(np.prod(alpha[b, :j])) for b in range(alpha.shape[0]) for j in range(W))
        return 1.0 - tot / alpha.size
    truth = 1.0 - expected_prefix_by_enumeration(a) / W
    assert abs(O.e2e_tv_loss(a, W) - truth) < 1e-14
    assert abs(bad_loss(a, W) - truth) > 1e-3


def test_interleaved_rope_breaks_closed_form():
    def bad_rope(x, pos, theta):
        x = np.asarray(x, dtype=np.float64)
        d = x.shape[-1]
        inv = theta ** (-2.0 * np.arange(d // 2) / d)
        ang = np.asarray(pos, np.float64)[:, None] * inv[None, :]
        c, s = np.cos(ang)[:, None, :], np.sin(ang)[:, None, :]
        x1, x2 = x[..., 0::2], x[..., 1::2]
        out = np.empty_like(x)
        out[..., 0::2] = x1 * c - x2 * s
        out[..., 1::2] = x2 * c + x1 * s
        return out
    x = np.zeros((1, 1, 4))
    x[0, 0, 0] = 1.0
    expect = [np.cos(3.0), 0.0, np.sin(3.0), 0.0]
    assert np.allclose(A.rope(x, np.array([3]), 1e4)[0, 0], expect)
    assert not np.allclose(bad_rope(x, np.array([3]), 1e4)[0, 0], expect)


def test_anchor_excluded_breaks_history_visibility():
    from tests.test_oracle_tree import history_visibility
    args = ([12], [3], [3], [4, 9, 6], 3)
    pt = T.pack(*args)
    good = T.dense_mask(pt)
    assert np.array_equal(good, history_visibility(*args))
    bad = good.copy()
    for b, rows in enumerate(pt.branch_rows):
        bad[rows, pt.anchors_global[b]] = False   # x_{<a_b} instead of x_{<=a_b}
    assert not np.array_equal(bad, history_visibility(*args))


def test_sibling_leak_breaks_causal_equivalence():
    pt = T.pack([10], [2], [2], [4, 4], 3)
    rng = np.random.default_rng(9)
    q = rng.standard_normal((pt.num_rows, 2, 8))
    k = rng.standard_normal((pt.num_rows, 1, 8))
    v = rng.standard_normal((pt.num_rows, 1, 8))
    ind = A.branch_causal_attention(pt, q, k, v, 1e4)
    orig = T.visible
    try:
        # leak: branch rows also see the sibling branch at the same anchor
        def leaky(p, r):
            cols = orig(p, r)
            b = int(p.branch_of[r])
            if b >= 0:
                other = p.branch_rows[1 - b]
                cols = np.asarray(sorted(set(cols.tolist()) | set(other)), np.int64)
            return cols
        T.visible = leaky
        bad = A.tree_attention(pt, q, k, v, 1e4)
    finally:
        T.visible = orig
    assert np.max(np.abs(bad - ind)) > 1e-3


def test_lm_head_slips_break_pins():
    """A head used untransposed, or q_less counted with <= instead of <,
    breaks the one-hot readout and the identical-model pins."""
    import pytest
    from oracle import lm_head as LM
    rng = np.random.default_rng(11)
    H, V = 6, 11
    head = rng.normal(size=(V, H))
    with pytest.raises(ValueError):  # h @ head cannot even be formed for H != V
        np.eye(H) @ head
    sq = rng.normal(size=(H, H))     # a square head: the untransposed product runs but is wrong
    assert not np.array_equal(np.eye(H) @ sq, sq.T)
    assert np.array_equal(LM.prediction_logits(np.eye(H), sq), sq.T)
    h = rng.normal(size=(4, H))
    z = h @ head.T
    q, active, log_q = O.draft_probs(z)
    _, log_p = O.teacher_probs(z)
    bad_q_less = (q * ((log_q <= log_p) & active)).sum(axis=-1)
    good = LM.row_statistics(z, z)["q_less"]
    assert np.all(good == 0.0) and np.all(np.abs(bad_q_less - 1.0) < 1e-12)


def test_gdn_decay_outside_the_correction_breaks_the_erase_pin():
    """S_t = alpha S - beta (S k) k^T + beta v k^T (decay not applied to the
    correction term) leaves -0.5 v1 k1^T where the true rule erases the key."""
    from oracle import gdn as G
    rng = np.random.default_rng(12)
    k1 = np.linalg.qr(rng.normal(size=(6, 6)))[0][:, 0]
    v1 = rng.normal(size=4)

    def slipped(k, v, alpha, beta):
        S = np.zeros((v.shape[1], k.shape[1]))
        for t in range(k.shape[0]):
            S = alpha[t] * S - beta[t] * np.outer(S @ k[t], k[t]) + beta[t] * np.outer(v[t], k[t])
        return S
    k = np.vstack([k1, k1])
    v = np.vstack([v1, np.zeros(4)])
    a, b = np.array([1.0, 0.5]), np.array([1.0, 1.0])
    _, S = G.gdn_sequence(k, k, v, a, b)
    assert np.max(np.abs(S)) < 1e-13
    assert np.max(np.abs(slipped(k, v, a, b))) > 0.1


def test_sparse_boundary_group_keyed_by_trunk_only_breaks_the_branch_pin():
    """Keying the group that a branch token completes by its trunk members only
    (not branch-specific) makes both branches pick the same group, which the
    branch-specific pin rules out."""
    from oracle import sparse as SP
    from oracle import tree as T

    def slipped(pt, r, qi, ki, g, topk, kvh):
        hist = SP.history(pt, r)
        n = (len(hist)) // g
        keys = []
        for m in range(n):
            members = [c for c in hist[m * g:(m + 1) * g] if pt.parent is not None and c < 12]  # trunk rows only
            keys.append(np.mean(ki[members, kvh], axis=0))
        scores = np.stack(keys) @ qi[r, kvh]
        best = sorted(range(n), key=lambda m: (-scores[m], m))[:topk]
        return [c for m in sorted(best) for c in hist[m * g:(m + 1) * g]]
    pt = T.pack([12], [0], [2], [6, 6], 2, True)
    qi = np.zeros((pt.num_rows, 1, 2))
    ki = np.zeros((pt.num_rows, 1, 2))
    qi[12, 0] = qi[14, 0] = [1.0, 0.0]
    ki[12, 0], ki[14, 0] = [10.0, 0.0], [-10.0, 0.0]
    ki[0:4, 0] = [0.5, 0.0]
    good = (SP.selected_columns(pt, 12, qi, ki, 4, 1, 0), SP.selected_columns(pt, 14, qi, ki, 4, 1, 0))
    bad = (slipped(pt, 12, qi, ki, 4, 1, 0), slipped(pt, 14, qi, ki, 4, 1, 0))
    assert good[0] != good[1]
    assert bad[0][:4] == bad[1][:4] == [0, 1, 2, 3]   # both branches fall back to the trunk group


def test_conv_over_packed_neighbours_breaks_the_fir_pin():
    """Convolving over the packed neighbours r, r-1, ... instead of the row's
    history puts a sibling's or trunk tail's tokens in a branch row's window;
    the per-history FIR pin catches it."""
    from scipy.signal import lfilter
    from oracle import conv as CV

    def slipped(pt, x, w):
        out = np.zeros_like(x)
        for r in range(pt.num_rows):
            for j in range(w.shape[1]):
                if r - j >= 0:
                    out[r] += w[:, j] * x[r - j]
        return out
    pt = T.pack([20], [3], [3], [5, 5, 19], 4, True)
    rng = np.random.default_rng(1)
    x = rng.normal(size=(pt.num_rows, 3))
    w = rng.normal(size=(3, 4))

    def fir_mismatch(conv):
        out = conv(pt, x, w)
        worst = 0.0
        for r in range(pt.num_rows):
            hist = CV.history(pt, r)
            ref = np.stack([lfilter(w[c], [1.0], x[hist, c]) for c in range(3)], axis=1)[-1]
            worst = max(worst, float(np.max(np.abs(out[r] - ref))))
        return worst
    assert fir_mismatch(CV.tree_causal_conv) < 1e-12
    assert fir_mismatch(slipped) > 0.1
