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


def test_tile_split_partitions_the_tiles_by_cost():
    anchors = np.array([40, 41, 60, 90, 95, 99, 10, 12, 30], np.int32)
    trunk, nbr, W = [100, 60], [6, 3], 8
    costs = PAR.tile_costs(trunk, nbr, anchors, W)
    rows = PAR.tile_rows(trunk, nbr, W)
    # brute force: visible pairs of every row, summed per tile
    per_row = []
    a = 0
    for T, B in zip(trunk, nbr):
        per_row += [j + 1 for j in range(T)]
        for b in range(B):
            per_row += [int(anchors[a + b]) + 1 + i for i in range(1, W + 1)]
        a += B
    assert rows[-1, 1] == len(per_row)
    assert [int(c) for c in costs] == [sum(per_row[r0:r1]) for r0, r1 in rows]
    for world in (1, 2, 3, 5):
        spans = [PAR.split_tiles(costs, world, r) for r in range(world)]
        assert spans[0][0] == 0 and spans[-1][1] == len(costs)
        assert all(spans[r][1] == spans[r + 1][0] for r in range(world - 1))
        if world <= len(costs):
            share = [costs[t0:t1].sum() for t0, t1 in spans]
            assert max(share) <= costs.sum() / world + costs.max()


def _split_rank_main(rank, world, port, out_dir):
    """One rank of the split step, the oracle standing in for the kernels: its
    run of query tiles (attention rows) and its share of whole branches
    (overlap, loss with the global count, gradient); the loss shares summed
    over the process group."""
    import synthetic as SY
    from oracle import attention as OA
    from oracle import tree as OT
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        case = SY.make_case("split", [(150, 20, 6), (90, 10, 4)], W=4, Hq=4, Hkv=2, d=16, dtype="f32", vocab=40,
                            sig_t=3.0, sig_n=1.0, seed=8)
        nb = int(sum(case.num_branches))
        costs = PAR.tile_costs(case.trunk_len, case.num_branches, case.anchors, case.W)
        t0, t1 = PAR.split_tiles(costs, world, rank)
        trows = PAR.tile_rows(case.trunk_len, case.num_branches, case.W)
        rows = list(range(int(trows[t0, 0]), int(trows[t1 - 1, 1]))) if t1 > t0 else []
        pt = OT.pack(case.trunk_len, case.prompt_len, case.num_branches, case.anchors, case.W, True)
        attn = OA.tree_attention(pt, case.q, case.k, case.v, theta=case.theta, rows=rows) if rows else \
            np.zeros((0, case.Hq, case.d))
        b0, b1 = PAR.shard_range(nb, world, rank)
        lr = slice(b0 * case.W, b1 * case.W)
        z, t = case.draft[lr].astype(np.float64), case.teacher[lr].astype(np.float64)
        count = nb * case.W
        loss = PAR.global_loss(OO.e2e_tv_loss(OO.overlap(z, t), case.W, count=count))
        grad = OO.e2e_tv_grad_draft(z, t, case.W, count=count)
        np.savez(os.path.join(out_dir, f"s{rank}.npz"), rows=np.asarray(rows, np.int64), attn=attn, loss=loss,
                 b0=b0, grad=grad)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_split_one_batch_end_to_end():
    import synthetic as SY
    from oracle import attention as OA
    from oracle import tree as OT
    world = 2
    with tempfile.TemporaryDirectory() as out_dir:
        mp.spawn(_split_rank_main, args=(world, _free_port(), out_dir), nprocs=world, join=True)
        res = [np.load(os.path.join(out_dir, f"s{r}.npz")) for r in range(world)]
    case = SY.make_case("split", [(150, 20, 6), (90, 10, 4)], W=4, Hq=4, Hkv=2, d=16, dtype="f32", vocab=40,
                        sig_t=3.0, sig_n=1.0, seed=8)
    pt = OT.pack(case.trunk_len, case.prompt_len, case.num_branches, case.anchors, case.W, True)
    full = OA.tree_attention(pt, case.q, case.k, case.v, theta=case.theta)
    rows = np.concatenate([r["rows"] for r in res])
    assert np.array_equal(rows, np.arange(pt.num_rows))       # every row scored exactly once
    np.testing.assert_allclose(np.concatenate([r["attn"] for r in res]), full, rtol=0, atol=1e-12)
    z, t = case.draft.astype(np.float64), case.teacher.astype(np.float64)
    full_loss = OO.e2e_tv_loss(OO.overlap(z, t), case.W)
    for r in res:
        assert abs(float(r["loss"]) - full_loss) <= 1e-12
    grad = np.concatenate([r["grad"] for r in sorted(res, key=lambda r: int(r["b0"]))])
    np.testing.assert_allclose(grad, OO.e2e_tv_grad_draft(z, t, case.W), rtol=1e-12, atol=1e-15)


def test_vocab_range_partitions_in_tile_blocks():
    for V in (1, 255, 256, 1000, 151936, 248320):
        for world in (1, 2, 3, 8):
            spans = [PAR.vocab_range(V, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == V
            assert all(spans[r][1] == spans[r + 1][0] for r in range(world - 1))
            assert all(lo % 256 == 0 or lo == hi == V for lo, hi in spans)   # empty shards sit at V


def _vocab_rank_main(rank, world, port, out_dir):
    """One rank of the vocabulary-parallel LM head, the oracle standing in for
    the three phases: log-sum-exps of its logit columns, gathered and merged;
    alpha / q_less shares with the global normalisers, gathered and summed;
    the loss from the merged alpha; dL/dz of its columns."""
    import synthetic as SY
    from oracle import lm_head as LM
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        case = SY.make_lm_head_case("vp", 2, 3, 700, 64, 64, sig_t=3.0, sig_n=1.0, seed=4)
        f = lambda a: SY.to_f64(a, "bf16")
        v0, v1 = PAR.vocab_range(case.V, world, rank)
        z = LM.prediction_logits(f(case.h_draft), f(case.w_draft)[v0:v1])
        t = LM.prediction_logits(f(case.h_teacher), f(case.w_teacher)[v0:v1])
        lse = lambda x: x.max(axis=1) + np.log(np.exp(x - x.max(axis=1, keepdims=True)).sum(axis=1))
        gz = PAR.gather_rows(torch.from_numpy(lse(z))).numpy()
        gt = PAR.gather_rows(torch.from_numpy(lse(t))).numpy()
        lz = np.logaddexp.reduce(gz, axis=0)
        lt = np.logaddexp.reduce(gt, axis=0)
        q, p = np.exp(z - lz[:, None]), np.exp(t - lt[:, None])
        alpha = PAR.gather_rows(torch.from_numpy(np.minimum(q, p).sum(axis=1))).numpy().sum(axis=0)
        qless = PAR.gather_rows(torch.from_numpy(np.where(q < p, q, 0.0).sum(axis=1))).numpy().sum(axis=0)
        loss = OO.e2e_tv_loss(alpha, case.W)
        g = OO.e2e_tv_grad_alpha(alpha, case.W)
        grad = g[:, None] * q * ((q < p).astype(np.float64) - qless[:, None])
        np.savez(os.path.join(out_dir, f"v{rank}.npz"), v0=v0, v1=v1, alpha=alpha, loss=loss, grad=grad)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_split_the_vocabulary():
    import synthetic as SY
    from oracle import lm_head as LM
    world = 2
    with tempfile.TemporaryDirectory() as out_dir:
        mp.spawn(_vocab_rank_main, args=(world, _free_port(), out_dir), nprocs=world, join=True)
        res = [np.load(os.path.join(out_dir, f"v{r}.npz")) for r in range(world)]
    case = SY.make_lm_head_case("vp", 2, 3, 700, 64, 64, sig_t=3.0, sig_n=1.0, seed=4)
    f = lambda a: SY.to_f64(a, "bf16")
    hd, wd, ht, wt = f(case.h_draft), f(case.w_draft), f(case.h_teacher), f(case.w_teacher)
    full = LM.lm_head_overlap(hd, wd, ht, wt, case.W)
    grad = OO.e2e_tv_grad_draft(LM.prediction_logits(hd, wd), LM.prediction_logits(ht, wt), case.W)
    for r in res:
        np.testing.assert_allclose(r["alpha"], full["alpha"], rtol=0, atol=1e-12)
        assert abs(float(r["loss"]) - full["loss"]) <= 1e-12
    got = np.concatenate([r["grad"] for r in sorted(res, key=lambda r: int(r["v0"]))], axis=1)
    np.testing.assert_allclose(got, grad, rtol=1e-10, atol=1e-14)


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
