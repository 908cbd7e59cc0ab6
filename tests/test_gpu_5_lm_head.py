"""Overlap statistics from hidden states and LM heads on the GPU against the
oracle: alpha, q_less and L within 1e-4 absolute, the normalisers within 1e-4
absolute, dL/dalpha within 1e-4 absolute, dL/dz within 1e-3 relative L2.  The
GPU forms the logits with bf16 products and fp32 accumulation; the oracle in
fp64 from the same bf16 values."""
import numpy as np
import pytest
import torch

import synthetic as SY
from oracle import lm_head as LM
from oracle import overlap as OO
from tree_attention_masked_b200 import specopd as S

pytestmark = pytest.mark.gpu

TOL = 1e-4
GRAD_TOL = 1e-3


def rel_l2(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def run(case, count=0.0, with_optional=True, with_grad=True):
    dev = torch.device("cuda")
    t = lambda a: torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
    hd, wd, ht, wt = t(case.h_draft), t(case.w_draft), t(case.h_teacher), t(case.w_teacher)
    R = case.rows
    f = lambda: torch.full((R,), float("nan"), device=dev)
    out = {"alpha": f(), "loss": torch.full((1,), float("nan"), device=dev)}
    if with_optional:
        out.update(q_less=f(), lse_draft=f(), lse_teacher=f(), grad_alpha=f())
    ws = torch.empty(S.specopd_lm_head_workspace_bytes(R, case.V), dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    grad = None
    if with_grad:  # rows padded to a multiple of 4 floats; the pad must stay untouched
        ld = (case.V + 3) // 4 * 4
        gbuf = torch.full((R, ld), 7.0, device=dev)
        grad = gbuf[:, :case.V]
    S.specopd_lm_head_overlap(hd, wd, ht, wt, case.num_branches, case.W, count, out["alpha"], out["loss"], ws,
                              status, q_less=out.get("q_less"), lse_draft=out.get("lse_draft"),
                              lse_teacher=out.get("lse_teacher"), grad_alpha=out.get("grad_alpha"), grad=grad)
    torch.cuda.synchronize()
    assert status.item() == 0
    res = {k: v.cpu().numpy().astype(np.float64) for k, v in out.items()}
    if with_grad:
        assert torch.all(gbuf[:, case.V:] == 7.0)
        res["grad"] = grad.cpu().numpy().astype(np.float64)
    return res


def oracle(case, rows=None, count=None):
    """The oracle's statistics, plus dL/dz (the overlap module's gradient on the
    oracle's logits).  rows: whole branches; count then defaults to all rows."""
    f64 = lambda a: SY.to_f64(a, "bf16")
    hd, ht = f64(case.h_draft), f64(case.h_teacher)
    if rows is not None:
        hd, ht = hd[rows], ht[rows]
        count = case.rows if count is None else count
    wd, wt = f64(case.w_draft), f64(case.w_teacher)
    out = LM.lm_head_overlap(hd, wd, ht, wt, case.W, count)
    out["grad"] = OO.e2e_tv_grad_draft(LM.prediction_logits(hd, wd), LM.prediction_logits(ht, wt), case.W, count)
    return out


CASES = [
    # name, branches, W, V, Hd, Ht
    ("tiny", 2, 4, 1000, 128, 128),        # one row tile, a ragged vocabulary tile
    ("ragged-rows", 5, 7, 777, 64, 64),    # 35 rows: a partial row tile; the smallest hidden size
    ("exact-tiles", 32, 8, 512, 128, 128),  # 256 rows and 512 entries: whole tiles only
    ("two-heads", 3, 16, 3000, 64, 192),   # different draft and teacher hidden sizes
    ("multi-tile", 24, 16, 8191, 256, 256),  # 3 row tiles x 32 vocabulary tiles, more tiles than some SMs take
    ("one-entry", 1, 1, 1, 64, 64),        # V = 1: q = p = 1, alpha = 1
]


@pytest.mark.parametrize("name,nb,W,V,Hd,Ht", CASES)
def test_lm_head_overlap_matches_oracle(name, nb, W, V, Hd, Ht):
    case = SY.make_lm_head_case(name, nb, W, V, Hd, Ht, sig_t=3.0, sig_n=1.5, seed=len(name))
    got = run(case)
    ref = oracle(case)
    keys = ["alpha", "q_less", "lse_draft", "lse_teacher", "grad_alpha"]
    if V == 1:
        # q = p = 1 exactly: a tie that fp32 rounding may settle either way.
        # Both q_less = 0 and 1 are valid subgradients of min there, and the
        # gradient q (bit - q_less) is 0 for both, so only the set is checked.
        keys.remove("q_less")
        assert set(got["q_less"].tolist()) <= {0.0, 1.0}
    for k in keys:
        assert np.max(np.abs(got[k] - ref[k])) <= TOL, (k, np.max(np.abs(got[k] - ref[k])))
    assert abs(got["loss"][0] - ref["loss"]) <= TOL
    if V == 1:
        assert np.max(np.abs(got["grad"])) <= 1e-6   # q (bit - q_less) = 0 for either tie decision
    else:
        assert rel_l2(got["grad"], ref["grad"]) <= GRAD_TOL, rel_l2(got["grad"], ref["grad"])


def test_identical_models_give_full_overlap():
    case = SY.make_lm_head_case("same", 4, 8, 5000, 128, 128, sig_t=3.0, sig_n=0.0, seed=3)
    assert np.array_equal(case.w_draft, case.w_teacher) and np.array_equal(case.h_draft, case.h_teacher)
    got = run(case)
    assert np.max(np.abs(got["alpha"] - 1.0)) <= 1e-5
    assert np.all(got["q_less"] == 0.0)   # identical logits: q < p nowhere
    assert abs(got["loss"][0]) <= 1e-5
    # q < p nowhere and q_less = 0: dL/dz = g q (0 - 0) = 0 exactly
    assert np.all(got["grad"] == 0.0)


def test_optional_outputs_and_count():
    case = SY.make_lm_head_case("opt", 3, 4, 2048, 64, 64, sig_t=2.0, sig_n=1.0, seed=9)
    a = run(case, with_optional=False, with_grad=False)
    b = run(case, count=100.0)
    assert np.array_equal(a["alpha"], b["alpha"])   # the same launches: identical bits
    ref = oracle(case, count=100)
    assert abs(b["loss"][0] - ref["loss"]) <= TOL


def test_repeatable_bits():
    case = SY.make_lm_head_case("rep", 8, 16, 4096, 128, 128, sig_t=3.0, sig_n=1.5, seed=5)
    a, b = run(case), run(case)
    for k in a:
        assert np.array_equal(a[k], b[k]), k


def test_full_size_sampled_branches():
    """The 8B-style shape: 1,024 prediction rows, hidden size 4,096, V = 151,936
    (594 vocabulary tiles, 8 row tiles); the oracle on three whole branches."""
    case = SY.make_lm_head_case("full", 64, 16, 151936, 4096, 4096, sig_t=3.0, sig_n=1.5, seed=0, workers=8)
    got = run(case)
    assert 0.0 <= got["loss"][0] <= 1.0
    for b in (0, 37, 63):
        rows = np.arange(b * 16, (b + 1) * 16)
        ref = oracle(case, rows=rows)
        for k in ("alpha", "q_less", "lse_draft", "lse_teacher", "grad_alpha"):
            assert np.max(np.abs(got[k][rows] - ref[k])) <= TOL, (b, k)
        assert rel_l2(got["grad"][rows], ref["grad"]) <= GRAD_TOL, b
    # the loss from the GPU's own alpha, by the definition
    from oracle import overlap as OO
    assert abs(got["loss"][0] - OO.e2e_tv_loss(got["alpha"], 16)) <= 1e-6


def test_vocabulary_shards_match_the_fused_call():
    """The vocabulary-parallel form, as ranks would run it, here one shard
    after another on one GPU: three shards of the heads' rows, phase 0 on each,
    the per-row log-sum-exps gathered (stacked in shard order) and merged,
    phase 1 on each with the global normalisers, the alpha / q_less shares
    merged, the E2E-TV loss on the merged alpha, phase 2 on each writing its
    columns of dL/dz.  Against the fused call and the fp64 oracle."""
    case = SY.make_lm_head_case("shards", 3, 5, 1800, 128, 192, sig_t=3.0, sig_n=1.5, seed=12)
    dev = torch.device("cuda")
    t = lambda a: torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
    hd, wd, ht, wt = t(case.h_draft), t(case.w_draft), t(case.h_teacher), t(case.w_teacher)
    R, V = case.rows, case.V
    cuts = [0, 512, 1536, V]
    shards = list(zip(cuts[:-1], cuts[1:]))
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    ws = [torch.empty(S.specopd_lm_head_workspace_bytes(R, v1 - v0), dtype=torch.uint8, device=dev)
          for v0, v1 in shards]
    f = lambda: torch.empty(R, device=dev)
    lz_p, lt_p = [f() for _ in shards], [f() for _ in shards]
    for k, (v0, v1) in enumerate(shards):
        S.specopd_lm_head_shard_phase(0, hd, wd[v0:v1], ht, wt[v0:v1], ws[k], status, lz_p[k], lt_p[k])
    lz2, lt2 = f(), f()
    S.specopd_merge_parts(torch.stack(lz_p), 1, lz2)
    S.specopd_merge_parts(torch.stack(lt_p), 1, lt2)
    a_p, q_p = [f() for _ in shards], [f() for _ in shards]
    for k, (v0, v1) in enumerate(shards):
        S.specopd_lm_head_shard_phase(1, hd, wd[v0:v1], ht, wt[v0:v1], ws[k], status, a_p[k], q_p[k], lz2=lz2,
                                      lt2=lt2)
    alpha, q_less = f(), f()
    S.specopd_merge_parts(torch.stack(a_p), 0, alpha)
    S.specopd_merge_parts(torch.stack(q_p), 0, q_less)
    loss, g = torch.empty(1, device=dev), f()
    S.specopd_e2e_tv_loss(alpha, case.num_branches, case.W, 0.0, loss, g)
    ld = (V + 3) // 4 * 4
    grad = torch.full((R, ld), 7.0, device=dev)
    for k, (v0, v1) in enumerate(shards):
        S.specopd_lm_head_shard_phase(2, hd, wd[v0:v1], ht, wt[v0:v1], ws[k], status, grad[:, v0:], lz2=lz2,
                                      q_less=q_less, grad_alpha=g)
    torch.cuda.synchronize()
    assert status.item() == 0
    assert torch.all(grad[:, V:] == 7.0)
    fused = run(case)
    got_a = alpha.cpu().numpy().astype(np.float64)
    assert np.max(np.abs(got_a - fused["alpha"])) <= 1e-5
    assert abs(loss.item() - fused["loss"][0]) <= 1e-5
    ref = oracle(case)
    assert np.max(np.abs(got_a - ref["alpha"])) <= TOL
    assert np.max(np.abs(q_less.cpu().numpy() - ref["q_less"])) <= TOL
    assert abs(loss.item() - ref["loss"]) <= TOL
    assert rel_l2(grad[:, :V].cpu().numpy().astype(np.float64), ref["grad"]) <= GRAD_TOL
    np.testing.assert_allclose(lz2.cpu().numpy() * np.log(2), ref["lse_draft"], rtol=0, atol=TOL)
