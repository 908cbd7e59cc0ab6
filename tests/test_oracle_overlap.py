"""Pins for the oracle's overlap, E2E-TV loss and gradient (CPU only).

What fixes the answers:
  * the worked example of the daiwk.github.io write-up (section "Checks,
    negative controls, and limits"), stored in tests/golden/worked_example.json;
  * sum_v min(q, p) = 1 - (1/2) ||p - q||_1 for two distributions (total
    variation identity);
  * prod-of-prefixes is the expected accepted-prefix length when draft token i
    is accepted independently with probability alpha_i: brute-force enumeration
    of the 2^W accept/reject patterns gives the same number;
  * central finite differences of the fp64 objective give the gradient;
  * closed cases: W = 1, all alpha = 1, all alpha = 0, p = q, disjoint supports.
"""
import itertools
import json
import os

import numpy as np
import pytest

from oracle import overlap as O

GOLD = os.path.join(os.path.dirname(__file__), "golden", "worked_example.json")


def test_worked_example():
    g = json.load(open(GOLD))
    q = np.asarray(g["draft_q"])
    p = np.asarray(g["teacher_p"])
    with np.errstate(divide="ignore"):
        z = np.log(q)[None, :]   # q = 0 -> -inf: outside the draft support
    t = np.log(p)[None, :]
    alpha = O.overlap(z, t)
    assert abs(alpha[0] - g["alpha"]) < 1e-15
    assert abs(O.e2e_tv_loss(alpha, g["W"]) - g["loss"]) < 1e-15
    # negative control: renormalising the teacher onto the draft support gives 0
    support = q > 0
    p_renorm = np.where(support, p, 0.0) / p[support].sum()
    assert abs(1.0 - np.minimum(q, p_renorm).sum() - g["loss_if_teacher_renormalised"]) < 1e-15


def test_worked_example_with_nan_padding():
    z = np.array([[np.log(.5), np.log(.5), np.nan]])
    t = np.log(np.array([[.4, .4, .2]]))
    assert abs(O.overlap(z, t)[0] - 0.8) < 1e-15


def test_total_variation_identity():
    rng = np.random.default_rng(0)
    z = rng.normal(0, 3, (20, 50))
    t = z + rng.normal(0, 1, (20, 50))
    z[3, :10] = np.nan
    z[4, 5] = -np.inf
    q = np.exp(z - np.nanmax(z, axis=1, keepdims=True))
    q = np.where(np.isfinite(z), q, 0.0)
    q /= q.sum(axis=1, keepdims=True)
    p = np.exp(t - t.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    tv = 0.5 * np.abs(p - q).sum(axis=1)
    assert np.max(np.abs(O.overlap(z, t) - (1.0 - tv))) < 1e-13


def test_alpha_range_symmetry_and_special_cases():
    rng = np.random.default_rng(1)
    z = rng.normal(0, 2, (30, 40))
    t = rng.normal(0, 2, (30, 40))
    a = O.overlap(z, t)
    assert np.all(a >= 0) and np.all(a <= 1)
    assert np.max(np.abs(a - O.overlap(t, z))) < 1e-14       # symmetric for full supports
    assert np.max(np.abs(O.overlap(t, t) - 1.0)) < 1e-14       # p = q
    assert np.max(np.abs(O.overlap(t + 3.7, t) - 1.0)) < 1e-14  # shift invariance of softmax
    # disjoint supports: draft on {0,1}, teacher mass there is exp(-1e4) = 0
    zz = np.array([[0.0, 0.0, np.nan, np.nan]])
    tt = np.array([[-1e4, -1e4, 0.0, 0.0]])
    assert O.overlap(zz, tt)[0] == 0.0
    # an empty draft support: alpha = 0, gradient 0
    ze = np.full((1, 4), np.nan)
    assert O.overlap(ze, tt)[0] == 0.0
    assert np.all(O.overlap_grad_draft(ze, tt) == 0.0)


def test_teacher_mass_outside_support_is_kept():
    # draft support is half the vocabulary; teacher mass outside it lowers alpha
    t = np.zeros((1, 6))
    z = np.array([[0.0, 0.0, 0.0, np.nan, np.nan, np.nan]])
    assert abs(O.overlap(z, t)[0] - 0.5) < 1e-15


def test_nonfinite_inputs():
    t = np.zeros((1, 4))
    with pytest.raises(O.NonFiniteError):
        O.overlap(np.zeros((1, 4)), np.array([[0.0, np.nan, 0.0, 0.0]]))
    with pytest.raises(O.NonFiniteError):
        O.overlap(np.zeros((1, 4)), np.array([[0.0, np.inf, 0.0, 0.0]]))
    with pytest.raises(O.NonFiniteError):
        O.overlap(np.array([[0.0, np.inf, 0.0, 0.0]]), t)


def expected_prefix_by_enumeration(alpha_row):
    W = len(alpha_row)
    total = 0.0
    for pattern in itertools.product([0, 1], repeat=W):
        prob = 1.0
        for a, acc in zip(alpha_row, pattern):
            prob *= a if acc else (1.0 - a)
        n = 0
        while n < W and pattern[n]:
            n += 1
        total += prob * n
    return total


def test_loss_is_expected_accepted_prefix():
    rng = np.random.default_rng(2)
    B, W = 5, 6
    alpha = rng.uniform(0, 1, B * W)
    exp_len = sum(expected_prefix_by_enumeration(alpha[b * W:(b + 1) * W]) for b in range(B))
    assert abs(O.e2e_tv_loss(alpha, W) - (1.0 - exp_len / (B * W))) < 1e-13


def test_loss_closed_cases_and_monotonicity():
    rng = np.random.default_rng(3)
    a1 = rng.uniform(0, 1, 17)
    assert abs(O.e2e_tv_loss(a1, 1) - (1.0 - a1.mean())) < 1e-15    # W = 1
    assert O.e2e_tv_loss(np.ones(12), 4) == 0.0
    assert O.e2e_tv_loss(np.zeros(12), 4) == 1.0
    assert O.e2e_tv_loss(np.zeros(0), 4) == 0.0                      # empty batch
    # an early mismatch costs more than a late one
    early = np.array([0.5, 1.0, 1.0, 1.0])
    late = np.array([1.0, 1.0, 1.0, 0.5])
    assert O.e2e_tv_loss(early, 4) > O.e2e_tv_loss(late, 4)
    # prefix products never increase along a branch
    a = rng.uniform(0, 1, 8)
    pref = np.cumprod(a)
    assert np.all(np.diff(pref) <= 0)


def test_grad_alpha_finite_differences():
    rng = np.random.default_rng(4)
    B, W = 3, 5
    a = rng.uniform(0.05, 0.95, B * W)
    g = O.e2e_tv_grad_alpha(a, W)
    h = 1e-6
    for n in range(a.size):
        ap, am = a.copy(), a.copy()
        ap[n] += h
        am[n] -= h
        fd = (O.e2e_tv_loss(ap, W) - O.e2e_tv_loss(am, W)) / (2 * h)
        assert abs(fd - g[n]) < 1e-8


@pytest.mark.parametrize("inactive", [False, True])
def test_grad_draft_finite_differences(inactive):
    rng = np.random.default_rng(5)
    B, W, V = 2, 3, 7
    t = rng.normal(0, 2, (B * W, V))
    z = t + rng.normal(0, 1, (B * W, V))
    if inactive:
        z[1, 2] = np.nan
        z[4, 0] = -np.inf
    g = O.e2e_tv_grad_draft(z, t, W)
    h = 1e-6
    for r in range(B * W):
        for u in range(V):
            if not np.isfinite(z[r, u]):
                assert g[r, u] == 0.0
                continue
            zp, zm = z.copy(), z.copy()
            zp[r, u] += h
            zm[r, u] -= h
            fd = (O.loss_from_logits(zp, t, W) - O.loss_from_logits(zm, t, W)) / (2 * h)
            assert abs(fd - g[r, u]) < 1e-8, (r, u, fd, g[r, u])


def test_grad_properties():
    rng = np.random.default_rng(6)
    t = rng.normal(0, 2, (6, 30))
    z = t + rng.normal(0, 1, (6, 30))
    da = O.overlap_grad_draft(z, t)
    assert np.max(np.abs(da.sum(axis=1))) < 1e-15 * 30 + 1e-16   # softmax shift invariance
    assert np.all(O.e2e_tv_grad_draft(t, t, 3) == 0.0)            # p = q: no gradient
    # teacher is fixed: perturbing t changes alpha, but the objective's gradient
    # is taken with respect to z only (the oracle exposes no teacher gradient)
    assert not hasattr(O, "e2e_tv_grad_teacher")


def test_bf16_inputs_promote_exactly():
    from synthetic import bf16_round, to_f64
    rng = np.random.default_rng(7)
    x = rng.normal(0, 3, (4, 64)).astype(np.float32)
    xb = bf16_round(x)
    xf = to_f64(xb, "bf16")
    # every bf16 value is exactly representable: round trip is the identity
    assert np.array_equal(bf16_round(xf.astype(np.float32)), xb)
    assert np.max(np.abs(xf - x)) <= np.max(np.abs(x)) * 2.0 ** -8
