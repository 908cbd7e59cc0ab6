"""Pins for the oracle's prediction logits and the statistics taken from them (CPU only).

What fixes the answers:
  * a one-hot hidden state e_k reads out column k of the head: the logits of
    the identity rows are the head transposed, exactly;
  * the logits of one row by brute force: a Python sum of products per entry;
  * log-sum-exp, alpha and q_less of tiny rows by brute force with math.fsum;
  * identical draft and teacher (same hidden states, same head): q = p, so
    alpha = 1, q_less = 0 (strict comparison), L = 0 and dL/dalpha_{b,i} =
    -(W - i + 1)/count (every prefix product is 1);
  * a zero teacher hidden state gives a uniform teacher p = 1/V;
  * alpha - q_less is the teacher mass where q >= p.
"""
import math

import numpy as np
import pytest

from oracle import lm_head as LM


def test_one_hot_rows_read_out_head_columns():
    rng = np.random.default_rng(1)
    H, V = 6, 11
    head = rng.normal(size=(V, H))
    assert np.array_equal(LM.prediction_logits(np.eye(H), head), head.T)


def test_logits_brute_force():
    rng = np.random.default_rng(2)
    h = rng.normal(size=(3, 5))
    head = rng.normal(size=(7, 5))
    got = LM.prediction_logits(h, head)
    for r in range(3):
        for v in range(7):
            ref = math.fsum(float(h[r, k]) * float(head[v, k]) for k in range(5))
            assert abs(got[r, v] - ref) < 1e-13


def test_shape_mismatch_rejected():
    with pytest.raises(ValueError):
        LM.prediction_logits(np.zeros((2, 3)), np.zeros((4, 5)))


def _brute_row(zr, tr):
    mz = max(zr)
    lz = mz + math.log(math.fsum(math.exp(x - mz) for x in zr))
    mt = max(tr)
    lt = mt + math.log(math.fsum(math.exp(x - mt) for x in tr))
    q = [math.exp(x - lz) for x in zr]
    p = [math.exp(x - lt) for x in tr]
    alpha = math.fsum(min(a, b) for a, b in zip(q, p))
    q_less = math.fsum(a for a, b in zip(q, p) if a < b)
    return lz, lt, alpha, q_less


def test_row_statistics_brute_force():
    rng = np.random.default_rng(3)
    H, V, R = 4, 9, 5
    hd, ht = rng.normal(size=(R, H)), rng.normal(size=(R, H))
    wd, wt = rng.normal(size=(V, H)), rng.normal(size=(V, H))
    out = LM.lm_head_overlap(hd, wd, ht, wt, W=R)
    z, t = hd @ wd.T, ht @ wt.T
    for r in range(R):
        lz, lt, a, ql = _brute_row(list(z[r]), list(t[r]))
        assert abs(out["lse_draft"][r] - lz) < 1e-12
        assert abs(out["lse_teacher"][r] - lt) < 1e-12
        assert abs(out["alpha"][r] - a) < 1e-13
        assert abs(out["q_less"][r] - ql) < 1e-13


def test_identical_models():
    rng = np.random.default_rng(4)
    W, nb, H, V = 4, 3, 8, 16
    h = rng.normal(size=(nb * W, H))
    head = rng.normal(size=(V, H))
    out = LM.lm_head_overlap(h, head, h, head, W)
    assert np.max(np.abs(out["alpha"] - 1.0)) < 1e-13
    assert np.all(out["q_less"] == 0.0)
    assert abs(out["loss"]) < 1e-13
    expect = np.tile(-(W - np.arange(W)) / (nb * W), nb)
    assert np.max(np.abs(out["grad_alpha"] - expect)) < 1e-13


def test_zero_teacher_state_is_uniform():
    rng = np.random.default_rng(5)
    H, V = 6, 10
    hd = rng.normal(size=(2, H))
    wd = rng.normal(size=(V, H))
    out = LM.lm_head_overlap(hd, wd, np.zeros((2, H)), rng.normal(size=(V, H)), W=2)
    z = hd @ wd.T
    q = np.exp(z - z.max(axis=1, keepdims=True))
    q /= q.sum(axis=1, keepdims=True)
    assert np.max(np.abs(out["alpha"] - np.minimum(q, 1.0 / V).sum(axis=1))) < 1e-14
    assert np.max(np.abs(out["lse_teacher"] - math.log(V))) < 1e-14


def test_alpha_minus_q_less_is_teacher_mass_where_q_not_below_p():
    rng = np.random.default_rng(6)
    hd, ht = rng.normal(size=(4, 5)), rng.normal(size=(4, 5))
    wd, wt = rng.normal(size=(12, 5)), rng.normal(size=(12, 5))
    out = LM.lm_head_overlap(hd, wd, ht, wt, W=4)
    z, t = hd @ wd.T, ht @ wt.T
    q = np.exp(z - out["lse_draft"][:, None])
    p = np.exp(t - out["lse_teacher"][:, None])
    assert np.max(np.abs(out["alpha"] - out["q_less"] - np.where(q >= p, p, 0.0).sum(axis=1))) < 1e-14
    assert np.all(out["q_less"] <= out["alpha"] + 1e-15)
