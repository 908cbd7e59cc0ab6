"""Gated DeltaNet over a proposal tree on the GPU (trunk pass with C = 64
checkpoints, then indexed replay per branch) against the oracle's plain
sequential recurrence over each row's history: relative L2 <= 1e-4 (fp32 state
on the GPU, fp64 in the oracle, the same bf16 inputs), and every row within
1e-3 so that one wrong row cannot hide in the whole-tensor figure."""
import numpy as np
import pytest
import torch

import synthetic as SY
from oracle import gdn as OG
from oracle import tree as OT
from tree_attention_masked_b200 import specopd as S

pytestmark = pytest.mark.gpu

TOL = 1e-4
ROW_TOL = 1e-3


def run(case):
    dev = torch.device("cuda")
    bf = lambda a: torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
    anchors = torch.from_numpy(case.anchors).to(dev)
    trees = S.Trees(case.trunk_len, case.prompt_len, case.num_branches, case.W, anchors, case.pack_terminal)
    q, k, v = bf(case.q), bf(case.k), bf(case.v)
    alpha = torch.from_numpy(case.alpha).to(dev)
    beta = torch.from_numpy(case.beta).to(dev)
    out = torch.full((case.num_rows, case.H, 128), float("nan"), device=dev)
    nbytes = S.specopd_gdn_workspace_bytes(trees, case.H)
    ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    S.specopd_gdn_tree(trees, q, k, v, alpha, beta, out, ws, status)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64), status.item(), ws, nbytes


def oracle_rows(case, rows=None):
    pt = OT.pack(case.trunk_len, case.prompt_len, case.num_branches, case.anchors, case.W, case.pack_terminal)
    f = lambda a: SY.to_f64(a, "bf16")
    q, k, v = f(case.q), f(case.k), f(case.v)
    a, b = case.alpha.astype(np.float64), case.beta.astype(np.float64)
    if rows is None:
        return OG.gdn_tree(pt, q, k, v, a, b)
    out = np.zeros((len(rows), case.H, 128))
    for n, r in enumerate(rows):
        hist = OT.ancestors(pt, r)[::-1] + [r]
        for h in range(case.H):
            o, _ = OG.gdn_sequence(q[hist, h], k[hist, h], v[hist, h], a[hist, h], b[hist, h])
            out[n, h] = o[-1]
    return out


def rel_l2(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def check(got, ref, rows=None):
    """Whole-tensor and per-row relative L2 of GPU rows `rows` (all rows by default)."""
    g = got if rows is None else got[rows]
    assert np.all(np.isfinite(g))
    assert rel_l2(g, ref) <= TOL, rel_l2(g, ref)
    per_row = [rel_l2(g[i], ref[i]) for i in range(g.shape[0])]
    worst = int(np.argmax(per_row))
    assert per_row[worst] <= ROW_TOL, (worst if rows is None else rows[worst], per_row[worst])


CASES = [
    dict(trees=[(40, 5, 3)], W=4, H=2),                       # trunk below one checkpoint interval
    dict(trees=[(200, 10, 6)], W=4, H=2, anchors=[[63, 127, 128, 10, 199, 64]]),  # anchors on and next to boundaries
    dict(trees=[(150, 20, 4), (70, 3, 2), (64, 0, 1)], W=3, H=1),  # several trees; a trunk of exactly 64
    dict(trees=[(130, 10, 5)], W=1, H=2),                     # one-token branches
    dict(trees=[(130, 10, 5)], W=5, H=2, pack_terminal=False),  # terminal rows not packed
    dict(trees=[(200, 10, 4)], W=20, H=2),                    # 20-sample branches: the 32-step branch solve
    dict(trees=[(150, 10, 3)], W=64, H=1),                    # 64-sample branches: the 64-step branch solve
    dict(trees=[(300, 50, 3)], W=40, H=1, pack_terminal=False),  # 39 rows per branch, padded to 64
]


@pytest.mark.parametrize("cfg", CASES)
def test_gdn_tree_matches_oracle(cfg):
    cfg = dict(cfg)
    anchors = cfg.pop("anchors", None)
    case = SY.make_gdn_case("gdn", cfg.pop("trees"), seed=7, anchors=anchors, **cfg)
    got, status, _, _ = run(case)
    assert status == 0
    check(got, oracle_rows(case))


def test_checkpoints_hold_the_boundary_states():
    case = SY.make_gdn_case("ck", [(192, 10, 2)], W=2, H=2, seed=3)
    _, status, ws, nbytes = run(case)
    assert status == 0
    ck = ws[:3 * 2 * 128 * 128 * 4].view(torch.float32).reshape(3, 2, 128, 128).cpu().numpy().astype(np.float64)
    f = lambda a: SY.to_f64(a, "bf16")
    ref = OG.checkpoint_states(f(case.q), f(case.k), f(case.v), case.alpha.astype(np.float64),
                               case.beta.astype(np.float64), 192, 64)
    assert rel_l2(ck, ref) <= TOL


def test_out_of_range_anchor_is_flagged_and_clamped():
    case = SY.make_gdn_case("bad", [(100, 20, 2)], W=2, H=1, seed=4, anchors=[[5, 99]])
    _, status, _, _ = run(case)
    assert status == 1   # SPECOPD_FLAG_ANCHOR


def test_full_size_sampled_rows():
    """The 8B-style tree (T = 4,096, 64 branches x W 16, 5,120 packed rows) with
    8 GDN heads; the oracle on trunk and branch rows from both ends."""
    case = SY.make_gdn_case("gdn-full", [(4096, 1024, 64)], W=16, H=8, seed=0)
    got, status, _, _ = run(case)
    assert status == 0
    rng = np.random.default_rng(5)
    rows = sorted({0, 63, 64, 4095, 4096, 4096 + 15, 4096 + 16 * 37 + 7, 5119} |
                  set(rng.choice(5120, size=16, replace=False).tolist()))
    check(got, oracle_rows(case, rows), rows)
