"""Host logic for several ranks (tree_attention_masked_b200.parallel).

Ranks score disjoint shares of one logical batch of branches with the global
prediction count (the write-up's section "Equations" normalises L by it), so
each rank's gradient rows are the global gradient's rows and the global loss
is sum_r L_r - (world - 1).  The CPU tests run two gloo ranks as separate
processes and check the recombination against the oracle on the whole
batch; the GPU test runs the fused C-ABI entry point on two shards of a batch
and checks them against one call on the whole batch.
"""
import os
import socket
import tempfile
from datetime import timedelta

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle.overlap as OO
from tree_attention_masked_b200 import parallel as PAR


def test_shard_range_is_a_partition():
    for n in (0, 1, 5, 64, 65, 1023):
        for world in (1, 2, 3, 8):
            ranges = [PAR.shard_range(n, world, r) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == n
            assert all(ranges[r][1] == ranges[r + 1][0] for r in range(world - 1))
            sizes = [hi - lo for lo, hi in ranges]
            assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 0
    for bad in ((4, 0, 0), (4, 2, 2), (4, 2, -1), (-1, 2, 0)):
        with pytest.raises(ValueError):
            PAR.shard_range(*bad)


def test_single_process_identities():
    assert PAR.global_count(48) == 48
    assert PAR.global_loss(0.25) == 0.25
    assert PAR.max_time_ms(3.5) == 3.5


B, W, V = 6, 3, 64


def _batch():
    rng = np.random.default_rng(5)  # the same logical batch on every rank
    z = rng.normal(size=(B * W, V)) * 2.0
    t = z + rng.normal(size=(B * W, V)) * 1.5
    z[:, -5:] = np.nan  # inactive draft padding, as in the pages' inputs
    return z, t


def _rank_main(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        z, t = _batch()
        lo, hi = PAR.shard_range(B, world, rank)
        rows = slice(lo * W, hi * W)
        count = PAR.global_count((hi - lo) * W)
        loss_local = OO.e2e_tv_loss(OO.overlap(z[rows], t[rows]), W, count=count)
        loss = PAR.global_loss(loss_local)
        grad = OO.e2e_tv_grad_draft(z[rows], t[rows], W, count=count)
        tmax = PAR.max_time_ms(1.5 + rank)
        np.savez(os.path.join(out_dir, f"r{rank}.npz"), loss=loss, tmax=tmax, count=count, lo=lo, hi=hi, grad=grad)
    finally:
        dist.destroy_process_group()


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_recombine_loss_and_gradient():
    world = 2
    with tempfile.TemporaryDirectory() as out_dir:
        mp.spawn(_rank_main, args=(world, _free_port(), out_dir), nprocs=world, join=True)
        res = [np.load(os.path.join(out_dir, f"r{r}.npz")) for r in range(world)]
    z, t = _batch()
    full_loss = OO.e2e_tv_loss(OO.overlap(z, t), W)
    full_grad = OO.e2e_tv_grad_draft(z, t, W)
    for r in res:
        assert int(r["count"]) == B * W
        assert float(r["tmax"]) == 1.5 + (world - 1)
        assert abs(float(r["loss"]) - full_loss) <= 1e-12
    grad = np.concatenate([r["grad"] for r in sorted(res, key=lambda r: int(r["lo"]))])
    assert grad.shape == full_grad.shape
    np.testing.assert_allclose(grad, full_grad, rtol=1e-12, atol=1e-15)


@pytest.mark.gpu
def test_branch_shards_on_gpu_recombine():
    """Two shards of one batch, each scored with the global count, against one
    call on the whole batch (same kernel, same rows: results agree to float
    rounding of the loss shares)."""
    import synthetic as SY
    from tests.gpu_cases import step_for
    from tree_attention_masked_b200 import specopd as S

    Bc, Wc, Vc = 6, 16, 151936
    case = SY.make_case("shards", [(Bc + 8, 2, Bc)], W=Wc, Hq=1, Hkv=1, d=32, dtype="bf16", vocab=Vc, sig_t=3.0,
                        sig_n=1.5, seed=33, inactive_frac=0.02)
    st = step_for(case)
    st.overlap()
    torch.cuda.synchronize()
    assert st.check_status() == 0
    full_alpha = st.alpha[:st.R].double().cpu().numpy()
    full_loss = float(st.loss.item())
    full_grad = st.grad.double().cpu().numpy()

    losses, alphas, grads = [], [], []
    for rank in range(2):
        lo, hi = PAR.shard_range(Bc, 2, rank)
        rows = slice(lo * Wc, hi * Wc)
        nr, nb = (hi - lo) * Wc, hi - lo
        alpha = torch.full((nr,), float("nan"), device="cuda")
        loss = torch.full((1,), float("nan"), device="cuda")
        grad = torch.full((nr, st.grad.stride(0)), float("nan"), device="cuda")[:, :Vc]
        ws = torch.empty(max(S.specopd_overlap_workspace_bytes(nr, Vc, nb), 256), dtype=torch.uint8, device="cuda")
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        S.specopd_tv_overlap_e2e(st.draft[rows], st.teacher[rows], Vc, nb, Wc, float(st.R), alpha, loss, grad, ws,
                                 status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        losses.append(float(loss.item()))
        alphas.append(alpha.double().cpu().numpy())
        grads.append(grad.double().cpu().numpy())
    np.testing.assert_array_equal(np.concatenate(alphas), full_alpha)
    np.testing.assert_array_equal(np.concatenate(grads), full_grad)
    assert abs(sum(losses) - 1.0 - full_loss) <= 1e-6
