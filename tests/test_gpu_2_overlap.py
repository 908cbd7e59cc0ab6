"""K4/K5 on the GPU against the oracle: alpha and L within 1e-4 absolute, the
gradient with respect to draft logits within 1e-3 relative L2."""
import numpy as np
import pytest
import torch

import synthetic as SY
from tests.gpu_cases import oracle_branch_grad, oracle_overlap, oracle_overlap_chunked, rel_l2, step_for
from oracle import overlap as OO

pytestmark = pytest.mark.gpu

ALPHA_TOL = 1e-4
GRAD_TOL = 1e-3


def overlap_case(B, W, V, dtype, sig_t=3.0, sig_n=1.0, inactive=0.0, seed=0):
    return SY.make_case("ov", [(max(B, 1) + 4, 2, B)], W=W, Hq=1, Hkv=1, d=32, dtype=dtype, vocab=V, sig_t=sig_t,
                        sig_n=sig_n, seed=seed, inactive_frac=inactive)


def run_overlap(case, with_grad=True):
    st = step_for(case, with_grad=with_grad)
    st.overlap()
    torch.cuda.synchronize()
    return st


SMALL = [
    (4, 4, 512, "f32", 0.0),
    (3, 5, 1000, "bf16", 0.0),         # V not a multiple of 8
    (2, 3, 37, "bf16", 0.0),           # tiny V
    (5, 1, 4099, "f32", 0.0),          # W = 1
    (4, 4, 20000, "bf16", 0.3),        # NaN-padded draft support
    (2, 8, 151936, "bf16", 0.0),       # full vocabulary of the 8B-style target
    (1, 16, 248320, "bf16", 0.05),     # 27B-scale vocabulary (16 CTAs per row)
    (3, 2, 70001, "f32", 0.0),
]


@pytest.mark.parametrize("B,W,V,dt,inact", SMALL, ids=[f"{s[0]}x{s[1]}x{s[2]}{s[3]}" for s in SMALL])
def test_overlap_loss_grad_small(B, W, V, dt, inact):
    case = overlap_case(B, W, V, dt, inactive=inact, seed=B * 7 + W)
    st = run_overlap(case)
    assert st.check_status() == 0
    a_ref = oracle_overlap(case)
    a = st.alpha.cpu().numpy()[:B * W].astype(np.float64)
    assert np.max(np.abs(a - a_ref)) <= ALPHA_TOL
    L_ref = OO.e2e_tv_loss(a_ref, W)
    assert abs(float(st.loss.item()) - L_ref) <= ALPHA_TOL
    g = st.grad.cpu().numpy().astype(np.float64)
    g_ref = np.concatenate([oracle_branch_grad(case, b, B * W) for b in range(B)])
    assert rel_l2(g, g_ref) <= GRAD_TOL
    if inact > 0:
        z = SY.to_f64(case.draft, case.dtype)
        assert np.all(g[~np.isfinite(z)] == 0.0)


def test_unfused_pieces_agree():
    case = overlap_case(3, 4, 3001, "bf16", seed=5)
    st = step_for(case)
    S = __import__("tree_attention_masked_b200.specopd", fromlist=["x"])
    R = st.R
    alpha = torch.empty(R, device="cuda")
    ql = torch.empty(R, device="cuda")
    lz = torch.empty(R, device="cuda")
    lt = torch.empty(R, device="cuda")
    S.specopd_tv_overlap(st.draft, st.teacher, st.vocab, alpha, ql, lz, lt, st.status)
    loss = torch.empty(1, device="cuda")
    ga = torch.empty(R, device="cuda")
    S.specopd_e2e_tv_loss(alpha, st.num_branches, st.W, 0.0, loss, ga)
    torch.cuda.synchronize()
    z = SY.to_f64(case.draft, "bf16")
    t = SY.to_f64(case.teacher, "bf16")
    a_ref = OO.overlap(z, t)
    assert np.max(np.abs(alpha.cpu().numpy() - a_ref)) <= ALPHA_TOL
    assert abs(loss.item() - OO.e2e_tv_loss(a_ref, 4)) <= ALPHA_TOL
    assert np.max(np.abs(ga.cpu().numpy() - OO.e2e_tv_grad_alpha(a_ref, 4))) <= 1e-5
    # natural-log normalisers
    zm = z.max(axis=1, keepdims=True)
    lz_ref = (zm + np.log(np.exp(z - zm).sum(axis=1, keepdims=True)))[:, 0]
    assert np.max(np.abs(lz.cpu().numpy() - lz_ref)) <= 1e-3
    q, _, _ = OO.draft_probs(z)
    p, _ = OO.teacher_probs(t)
    assert np.max(np.abs(ql.cpu().numpy() - (q * (q < p)).sum(axis=1))) <= ALPHA_TOL


def test_worked_example_on_gpu():
    # q = [.5,.5,0] (third entry outside the draft support), p = [.4,.4,.2]
    V = 8
    z = np.full((1, V), np.nan, np.float32)
    t = np.full((1, V), -1e4, np.float32)
    z[0, :2] = 0.0
    t[0, :3] = np.log(np.array([0.4, 0.4, 0.2], np.float32))
    case = SY.make_case("we", [(3, 0, 1)], W=1, Hq=1, Hkv=1, d=32, dtype="f32", vocab=V, anchors=[1])
    case.draft, case.teacher = z, t
    st = run_overlap(case)
    assert abs(st.alpha[0].item() - 0.8) <= 1e-6
    assert abs(st.loss.item() - 0.2) <= 1e-6


def test_nonfinite_teacher_flagged():
    case = overlap_case(2, 2, 100, "f32", seed=1)
    case.teacher[1, 17] = np.inf
    st = run_overlap(case)
    assert st.check_status() & 2


def test_empty_support_row():
    case = overlap_case(1, 2, 64, "f32", seed=2)
    case.draft[0, :] = np.nan
    st = run_overlap(case)
    assert st.alpha[0].item() == 0.0
    assert torch.all(st.grad[0] == 0)


def test_deterministic():
    case = overlap_case(6, 4, 30000, "bf16", seed=9)
    st = run_overlap(case)
    a1, l1, g1 = st.alpha.clone(), st.loss.clone(), st.grad.clone()
    st.overlap()
    torch.cuda.synchronize()
    assert torch.equal(a1, st.alpha) and torch.equal(l1, st.loss) and torch.equal(g1, st.grad)


@pytest.mark.parametrize("wl", [2, 3])
def test_overlap_full_size(wl):
    case = SY.make_workload(wl, workers=8)
    st = run_overlap(case)
    assert st.check_status() == 0
    a_ref = oracle_overlap_chunked(case)
    a = st.alpha.cpu().numpy()[:st.R].astype(np.float64)
    assert np.max(np.abs(a - a_ref)) <= ALPHA_TOL
    assert abs(float(st.loss.item()) - OO.e2e_tv_loss(a_ref, case.W)) <= ALPHA_TOL
    rng = np.random.default_rng(wl)
    nb = st.num_branches
    for b in sorted(set(rng.choice(nb, size=3, replace=False).tolist()) | {nb - 1}):
        g = st.grad[b * case.W:(b + 1) * case.W].cpu().numpy().astype(np.float64)
        assert rel_l2(g, oracle_branch_grad(case, b, st.R)) <= GRAD_TOL


@pytest.mark.parametrize("wl", [4, 5])
def test_overlap_full_size_sampled(wl):
    case = SY.make_workload(wl, workers=8)
    st = run_overlap(case)
    assert st.check_status() == 0
    rng = np.random.default_rng(wl)
    nb = st.num_branches
    L = float(st.loss.item())
    assert 0.0 <= L <= 1.0
    for b in sorted(set(rng.choice(nb, size=2, replace=False).tolist()) | {nb - 1}):
        rows = np.arange(b * case.W, (b + 1) * case.W)
        a = st.alpha.cpu().numpy()[rows].astype(np.float64)
        assert np.max(np.abs(a - oracle_overlap(case, rows))) <= ALPHA_TOL
        g = st.grad[b * case.W:(b + 1) * case.W].cpu().numpy().astype(np.float64)
        assert rel_l2(g, oracle_branch_grad(case, b, st.R)) <= GRAD_TOL
