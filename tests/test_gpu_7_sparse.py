"""Sparse attention with branch-consistent indexer groups on the GPU against the
fp64 oracle (the listing's Fig 4; readings in oracle/sparse.py).

The selection is an integer decision the kernel takes in fp32.  The test reads
the kernel's chosen groups back and checks them against the oracle's fp64
top-k: a chosen set may differ from the fp64 one only by swapping groups whose
fp64 scores lie within fp32 rounding of each other.  The bound used is the
standard one for the kernel's arithmetic: a group key is a sequential fp32 sum
of g exactly representable bf16 keys, divided by g (error <= gamma_g * mean|k|
per element), and the score di products summed in a fixed order with at most
di roundings on any path (error <= gamma_di * sum |q| |key|, whatever the
order), with gamma_n = n u / (1 - n u) and
u = 2^-24, so |score_fp32 - score| <= (gamma_di + gamma_g + gamma_di gamma_g)
* sum_e |q_e| mean_j |k_je|.  Rows whose set differs validly are compared
against the oracle's attention over the kernel's set; every other row against
the plain fp64 oracle.  Attention: relative L2 <= 1e-2 over the checked rows
and <= 2e-2 for every row (the dense tree attention's bars)."""
import numpy as np
import pytest
import torch

import synthetic as SY
from oracle import sparse as OS
from oracle import tree as OT
from tree_attention_masked_b200 import specopd as S

pytestmark = pytest.mark.gpu

TOL = 1e-2
ROW_TOL = 2e-2
THETA = 1e4
U32 = 2.0 ** -24


def gamma(n: int) -> float:
    return n * U32 / (1 - n * U32)


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
    sel = torch.full((N, case.Hkv, topk), -7, **i32)
    ws = torch.empty(S.specopd_sparse_workspace_bytes(trees, case.Hq, case.Hkv, case.di, g, topk),
                     dtype=torch.uint8, device=dev)
    S.specopd_sparse_tree_attention(trees, bf(case.q), bf(case.k), bf(case.v), bf(case.qi), bf(case.ki), out, pos,
                                    trunk_limit, anc_bits, tile_meta, g, topk, THETA, ws, status, selected=sel)
    torch.cuda.synchronize()
    return out.float().cpu().numpy().astype(np.float64), sel.cpu().numpy(), status.item()


def packed(case):
    return OT.pack(case.trunk_len, case.prompt_len, case.num_branches, case.anchors, case.W, case.pack_terminal)


def check_selection(case, pt, sel, g, topk, rows):
    """Returns {(row, kvh): kernel groups} for the rows whose set validly
    differs from the fp64 top-k; fails on any invalid set."""
    f = lambda a: SY.to_f64(a, "bf16")
    qi, ki = f(case.qi), f(case.ki)
    coef = gamma(case.di) + gamma(g) + gamma(case.di) * gamma(g)
    differ = {}
    for r in rows:
        hist = OS.history(pt, r)
        nc = len(hist) // g
        for kvh in range(case.Hkv):
            got = [int(x) for x in sel[r, kvh] if x >= 0]
            assert all(x == -1 for x in sel[r, kvh][len(got):]), (r, kvh, sel[r, kvh])
            assert got == sorted(got) and len(set(got)) == len(got), (r, kvh, got)
            assert len(got) == min(nc, topk), (r, kvh, got, nc)
            if nc == 0:
                continue
            s = OS.group_scores(pt, r, qi, ki, g, kvh)
            want = OS.top_groups(s, topk)
            if got == want:
                continue
            amag = np.stack([np.mean(np.abs(ki[hist[m * g:(m + 1) * g], kvh]), axis=0) for m in range(nc)])
            bound = coef * (amag @ np.abs(qi[r, kvh]))
            for m in set(got) - set(want):
                for mp in set(want) - set(got):
                    assert s[mp] - s[m] <= bound[m] + bound[mp], (r, kvh, m, mp, s[mp] - s[m], bound[m] + bound[mp])
            differ[(r, kvh)] = got
    return differ


def check(case, g, topk, rows=None):
    got, sel, status = run(case, g, topk)
    assert status == 0
    pt = packed(case)
    rows = list(range(pt.num_rows)) if rows is None else list(rows)
    differ = check_selection(case, pt, sel, g, topk, rows)
    # only near-ties may differ: a handful of (row, KV head) items at most
    assert len(differ) <= max(2, len(rows) * case.Hkv // 100), len(differ)
    f = lambda a: SY.to_f64(a, "bf16")
    ref = OS.sparse_tree_attention(pt, f(case.q), f(case.k), f(case.v), f(case.qi), f(case.ki), g, topk, THETA,
                                   rows=rows, selections=differ)
    out = got[rows]
    assert np.all(np.isfinite(out))
    err = float(np.linalg.norm(out - ref) / np.linalg.norm(ref))
    assert err <= TOL, err
    per_row = [float(np.linalg.norm(out[i] - ref[i]) / np.linalg.norm(ref[i])) for i in range(len(rows))]
    worst = int(np.argmax(per_row))
    assert per_row[worst] <= ROW_TOL, (rows[worst], per_row[worst])
    return sel


CASES = [
    # trees, W, Hq, Hkv, di, g, topk[, pack_terminal]
    # SIMT attention (g not a multiple of 64)
    ([(40, 5, 3)], 4, 2, 1, 16, 4, 2),                 # short trunk: few groups, tails everywhere
    ([(130, 10, 6), (70, 3, 2)], 5, 4, 2, 32, 8, 3),   # two trees, branch-completed boundary groups
    ([(130, 10, 5)], 1, 2, 2, 16, 3, 4),               # one-token branches; g does not divide the anchors
    ([(130, 10, 5)], 5, 2, 1, 16, 4, 64),              # k above the group count: dense tree attention
    ([(130, 10, 5)], 5, 2, 1, 24, 5, 2, False),        # terminal rows not packed
    # tensor cores (g a multiple of 64)
    ([(300, 40, 9)], 4, 4, 2, 32, 64, 2),              # 4 trunk groups, top-2, ragged last tile
    ([(700, 100, 12)], 16, 4, 1, 32, 64, 3),           # W = 16: branches complete boundary groups
    ([(129, 0, 5), (77, 70, 3), (400, 100, 17)], 3, 10, 2, 16, 64, 2),   # 3 trees, G = 5 (tile pairs)
    ([(700, 100, 12)], 8, 4, 2, 32, 128, 2),           # g = 128: one group per key block
    ([(300, 40, 9)], 4, 4, 2, 32, 64, 64),             # k above the group count: dense tree attention
    ([(300, 40, 9)], 4, 4, 2, 32, 64, 1, False),       # top-1, terminal rows not packed
]


@pytest.mark.parametrize("cfg", CASES, ids=range(len(CASES)))
def test_sparse_matches_oracle(cfg):
    trees, W, Hq, Hkv, di, g, topk = cfg[:7]
    ptf = cfg[7] if len(cfg) > 7 else True
    case = SY.make_sparse_case("sp", trees, W, Hq, Hkv, di, seed=3, pack_terminal=ptf)
    check(case, g, topk)


def test_dense_when_every_group_is_selected():
    """With k above every row's group count the sparse path is the tree
    attention: identical output to specopd_tree_attention on the same inputs."""
    from tests.gpu_cases import step_for
    case = SY.make_sparse_case("sp-dense", [(300, 40, 9)], 4, 4, 2, 32, seed=5)
    got, _, status = run(case, 64, 64)
    assert status == 0
    st = step_for(SY.Case(name="dense", trunk_len=case.trunk_len, prompt_len=case.prompt_len,
                          num_branches=case.num_branches, anchors=case.anchors, W=case.W, Hq=case.Hq,
                          Hkv=case.Hkv, d=128, dtype="bf16", theta=THETA, q=case.q, k=case.k, v=case.v,
                          draft=None, teacher=None, vocab=0, pack_terminal=True), with_grad=False)
    st.build_mask()
    st.attention()
    torch.cuda.synchronize()
    dense = st.out.float().cpu().numpy().astype(np.float64)
    assert np.array_equal(got, dense)


def test_full_size_sampled_rows():
    """The 8B-style tree (T = 4,096, 64 branches x W 16) with 32/8 heads,
    64-token groups, top-8 and 64-wide indexer features (tensor-core path);
    sampled trunk and branch rows, plus every row's selection of 256 sampled
    rows."""
    case = SY.make_sparse_case("sp-full", [(4096, 1024, 64)], 16, 32, 8, 64, seed=0)
    rng = np.random.default_rng(11)
    rows = sorted({0, 63, 64, 1000, 4095, 4096, 4096 + 15, 4096 + 16 * 37 + 9, 5119} |
                  set(rng.choice(5120, size=23, replace=False).tolist()))
    sel = check(case, 64, 8, rows)
    pt = packed(case)
    more = sorted(set(rng.choice(5120, size=256, replace=False).tolist()) - set(rows))
    check_selection(case, pt, sel, 64, 8, more)
