"""Sparse attention with branch-consistent indexer groups on the GPU against the
oracle.  The selection (an integer decision) is taken by both sides in the
kernel's precision: the oracle's scores in fp32 in the kernel's order
(decide_fp32); the attention itself is fp64 in the oracle and compared at the
bf16 output's tolerance, relative L2 <= 1e-2 (the dense tree attention's bar)."""
import numpy as np
import pytest
import torch

import synthetic as SY
from oracle import sparse as OS
from oracle import tree as OT
from tree_attention_masked_b200 import specopd as S

pytestmark = pytest.mark.gpu

TOL = 1e-2
THETA = 1e4


def run(case, g, topk):
    dev = torch.device("cuda")
    bf = lambda a: torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
    anchors = torch.from_numpy(case.anchors).to(dev)
    trees = S.Trees(case.trunk_len, case.prompt_len, case.num_branches, case.W, anchors, case.pack_terminal)
    N = case.num_rows
    i32 = dict(dtype=torch.int32, device=dev)
    pos, trunk_limit, branch_of = (torch.empty(N, **i32) for _ in range(3))
    anc_bits = torch.empty(N, dtype=torch.int64, device=dev)
    pred_rows = torch.empty(max(int(sum(case.num_branches)) * case.W, 1), **i32)
    cu_rows = torch.empty(len(case.trunk_len) + 1, **i32)
    tile_meta = torch.empty(max(S.specopd_tree_num_tiles(trees), 1), 8, **i32)
    status = torch.zeros(1, **i32)
    S.specopd_build_tree_mask(trees, pos, trunk_limit, branch_of, anc_bits, pred_rows, cu_rows, tile_meta, status)
    out = torch.empty(N, case.Hq, 128, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(S.specopd_sparse_workspace_bytes(trees, case.Hq, case.Hkv, case.di, g), dtype=torch.uint8,
                     device=dev)
    S.specopd_sparse_tree_attention(trees, bf(case.q), bf(case.k), bf(case.v), bf(case.qi), bf(case.ki), out, pos,
                                    g, topk, THETA, ws, status)
    torch.cuda.synchronize()
    return out.float().cpu().numpy().astype(np.float64), status.item()


def oracle(case, g, topk, rows=None):
    pt = OT.pack(case.trunk_len, case.prompt_len, case.num_branches, case.anchors, case.W, case.pack_terminal)
    f = lambda a: SY.to_f64(a, "bf16")
    return OS.sparse_tree_attention(pt, f(case.q), f(case.k), f(case.v), f(case.qi), f(case.ki), g, topk, THETA,
                                    rows=rows, decide_fp32=True)


def rel_l2(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


CASES = [
    # trees, W, Hq, Hkv, di, g, topk
    ([(40, 5, 3)], 4, 2, 1, 16, 4, 2),                 # short trunk: few groups, tails everywhere
    ([(130, 10, 6), (70, 3, 2)], 5, 4, 2, 32, 8, 3),   # two trees, branch-completed boundary groups
    ([(130, 10, 5)], 1, 2, 2, 16, 3, 4),               # one-token branches; g does not divide the anchors
    ([(130, 10, 5)], 5, 2, 1, 16, 4, 64),              # k above the group count: dense tree attention
    ([(130, 10, 5)], 5, 2, 1, 24, 5, 2, False),        # terminal rows not packed
]


@pytest.mark.parametrize("cfg", CASES)
def test_sparse_matches_oracle(cfg):
    trees, W, Hq, Hkv, di, g, topk = cfg[:7]
    ptf = cfg[7] if len(cfg) > 7 else True
    case = SY.make_sparse_case("sp", trees, W, Hq, Hkv, di, seed=3, pack_terminal=ptf)
    got, status = run(case, g, topk)
    assert status == 0
    ref = oracle(case, g, topk)
    assert rel_l2(got, ref) <= TOL, rel_l2(got, ref)


def test_full_size_sampled_rows():
    """The 8B-style tree (T = 4,096, 64 branches x W 16) with 32/8 heads,
    64-token groups, top-8 and 64-wide indexer features; sampled trunk and
    branch rows."""
    case = SY.make_sparse_case("sp-full", [(4096, 1024, 64)], 16, 32, 8, 64, seed=0)
    got, status = run(case, 64, 8)
    assert status == 0
    rows = [0, 63, 64, 1000, 4095, 4096, 4096 + 15, 4096 + 16 * 37 + 9, 5119]
    ref = oracle(case, 64, 8, rows=rows)
    assert rel_l2(got[rows], ref) <= TOL, rel_l2(got[rows], ref)
