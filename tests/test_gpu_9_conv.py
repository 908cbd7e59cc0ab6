"""The causal convolution along tree ancestry on the GPU against the fp64
oracle (oracle/conv.py; the listing's Fig 5).

fp32: every element within 1e-5 relative (+1e-6 absolute) of the oracle.
bf16: the output is the fp32 result rounded once to bf16, so every element
within 2^-8 relative (+1e-5 absolute)."""
import numpy as np
import pytest
import torch

import synthetic as SY
from oracle import conv as CV
from oracle import tree as OT
from tree_attention_masked_b200 import specopd as S

pytestmark = pytest.mark.gpu


def run(case, silu):
    from tree_attention_masked_b200.build import build
    build()
    dev = torch.device("cuda")
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
    if case.dtype == "bf16":
        x = torch.from_numpy(case.x.view(np.int16)).to(dev).view(torch.bfloat16)
    else:
        x = torch.from_numpy(case.x).to(dev)
    out = torch.full_like(x, float("nan"))
    S.specopd_tree_causal_conv(x, out, torch.from_numpy(case.weight).to(dev), torch.from_numpy(case.bias).to(dev),
                               pos, trunk_limit, cu_rows, silu=silu)
    torch.cuda.synchronize()
    assert status.item() == 0
    return out.float().cpu().numpy().astype(np.float64)


def check(case, silu, rows=None):
    got = run(case, silu)
    pt = OT.pack(case.trunk_len, case.prompt_len, case.num_branches, case.anchors, case.W, case.pack_terminal)
    x = SY.to_f64(case.x, case.dtype)
    rows = list(range(pt.num_rows)) if rows is None else list(rows)
    ref = CV.tree_causal_conv(pt, x, case.weight, case.bias, silu, rows=rows)
    rel, ab = (1e-5, 1e-6) if case.dtype == "f32" else (2.0 ** -8, 1e-5)
    err = np.abs(got[rows] - ref)
    assert np.all(err <= rel * np.abs(ref) + ab), float(np.max(err / (np.abs(ref) + ab)))


CASES = [
    # trees, W, C, Kw, dtype, silu, pack_terminal
    ([(100, 10, 4)], 4, 16, 4, "f32", False, True),
    ([(100, 10, 4)], 4, 16, 4, "bf16", True, True),
    ([(70, 3, 5), (40, 5, 2), (130, 30, 6)], 6, 24, 8, "bf16", False, True),   # three trees, wide window
    ([(64, 0, 6)], 1, 8, 3, "bf16", True, True),                             # one-sample branches
    ([(90, 20, 5)], 5, 32, 1, "f32", False, True),                           # width one
    ([(90, 20, 5)], 5, 384, 4, "bf16", True, False),                         # terminal rows not packed; C = 3 x 128
]


@pytest.mark.parametrize("cfg", CASES, ids=range(len(CASES)))
def test_conv_matches_oracle(cfg):
    trees, W, C, Kw, dtype, silu, ptf = cfg
    case = SY.make_conv_case("cv", trees, W, C, Kw, dtype=dtype, seed=7, pack_terminal=ptf)
    check(case, silu)


def test_full_size_tree_sampled_rows():
    """The 8B-style tree (T = 4,096, 64 branches x W 16) with 32 heads of 128
    channels (C = 4,096), width 4, SiLU; sampled trunk and branch rows."""
    case = SY.make_conv_case("cv-full", [(4096, 1024, 64)], 16, 4096, 4, seed=0)
    rng = np.random.default_rng(3)
    rows = sorted({0, 1, 2, 3, 4095, 4096, 4097, 4096 + 15, 5119} | set(rng.choice(5120, 40, replace=False).tolist()))
    check(case, True, rows)
