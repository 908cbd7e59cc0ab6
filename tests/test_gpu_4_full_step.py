"""The whole scoring step (mask -> RoPE + tree attention -> overlap, E2E-TV,
gradient) through the C ABI, against the oracle, on the tiny fp32 workload and
a small bf16 batch; and bitwise reproducibility of a full step."""
import numpy as np
import pytest
import torch

import synthetic as SY
from oracle import overlap as OO
from oracle import tree as OT
from tests.gpu_cases import oracle_attention_rows, oracle_branch_grad, packed, rel_l2, step_for, to_np

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("which", ["tiny-fp32", "small-bf16"])
def test_full_step_matches_oracle(which):
    if which == "tiny-fp32":
        case = SY.make_workload(1)
        tol = 1e-5
    else:
        case = SY.make_case("small", [(400, 100, 12), (260, 60, 5)], W=6, Hq=8, Hkv=2, d=128, dtype="bf16",
                            vocab=5000, sig_t=3.0, sig_n=1.5, seed=11)
        tol = 1e-2
    st = step_for(case)
    st.run()
    torch.cuda.synchronize()
    assert st.check_status() == 0
    pt = packed(case)
    assert np.array_equal(st.pred_rows.cpu().numpy()[:st.R], OT.prediction_rows(pt))
    ref = oracle_attention_rows(case, pt, range(pt.num_rows))
    assert rel_l2(to_np(st.out).astype(np.float64), ref) <= tol
    z = SY.to_f64(case.draft, case.dtype)
    t = SY.to_f64(case.teacher, case.dtype)
    a_ref = OO.overlap(z, t)
    assert np.max(np.abs(st.alpha.cpu().numpy()[:st.R] - a_ref)) <= 1e-4
    assert abs(st.loss.item() - OO.e2e_tv_loss(a_ref, case.W)) <= 1e-4
    g_ref = np.concatenate([oracle_branch_grad(case, b, st.R) for b in range(st.num_branches)])
    assert rel_l2(st.grad.cpu().numpy().astype(np.float64), g_ref) <= 1e-3


def test_full_step_bitwise_reproducible():
    case = SY.make_case("rep", [(600, 100, 16)], W=8, Hq=8, Hkv=2, d=128, dtype="bf16", vocab=20000, seed=12)
    st = step_for(case)
    st.run()
    torch.cuda.synchronize()
    snap = [x.clone() for x in (st.out, st.alpha, st.loss, st.grad, st.tile_meta)]
    for _ in range(2):
        st.run()
    torch.cuda.synchronize()
    for a, b in zip(snap, (st.out, st.alpha, st.loss, st.grad, st.tile_meta)):
        assert torch.equal(a, b)


def test_split_step_covers_the_batch():
    """The step as ranks of a split batch run it, here one share after another
    on one GPU: attention over three cost-balanced runs of query tiles (the
    query rows of each run and every key row rotated separately; odd G, so
    tile pairs shift at the run boundaries), the overlap over three shares of
    whole branches normalised by the whole batch's count.  Together they give
    the whole batch's outputs; the loss shares add up to the whole loss."""
    from tree_attention_masked_b200 import parallel as PAR
    case = SY.make_case("split", [(700, 100, 14), (300, 40, 6)], W=6, Hq=10, Hkv=2, d=128, dtype="bf16",
                        vocab=5000, sig_t=3.0, sig_n=1.5, seed=13)
    st = step_for(case)
    st.build_mask()
    world = 3
    costs = PAR.tile_costs(case.trunk_len, case.num_branches, case.anchors, case.W)
    trows = PAR.tile_rows(case.trunk_len, case.num_branches, case.W)
    assert len(costs) == st.num_tiles
    st.out.fill_(float("nan"))
    losses = []
    for rank in range(world):
        t0, t1 = PAR.split_tiles(costs, world, rank)
        if t1 > t0:
            st.attention(tiles=(t0, t1), rows=(int(trows[t0, 0]), int(trows[t1 - 1, 1])))
        b0, b1 = PAR.shard_range(st.num_branches, world, rank)
        st.overlap(count=float(st.R), branches=(b0, b1))
        torch.cuda.synchronize()
        losses.append(st.loss.item())
    assert st.check_status() == 0
    pt = packed(case)
    ref = oracle_attention_rows(case, pt, range(pt.num_rows))
    got = to_np(st.out).astype(np.float64)
    assert np.all(np.isfinite(got))                      # every row written by exactly one run
    assert rel_l2(got, ref) <= 1e-2
    assert max(rel_l2(got[r], ref[r]) for r in range(pt.num_rows)) <= 2e-2
    z = SY.to_f64(case.draft, case.dtype)
    t = SY.to_f64(case.teacher, case.dtype)
    a_ref = OO.overlap(z, t)
    assert np.max(np.abs(st.alpha.cpu().numpy()[:st.R] - a_ref)) <= 1e-4
    assert abs(sum(losses) - (world - 1) - OO.e2e_tv_loss(a_ref, case.W)) <= 1e-4
    g_ref = np.concatenate([oracle_branch_grad(case, b, st.R) for b in range(st.num_branches)])
    assert rel_l2(st.grad.cpu().numpy().astype(np.float64), g_ref) <= 1e-3
