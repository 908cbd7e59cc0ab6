"""K1 on the GPU against the oracle: positions, trunk limits, branch ids,
ancestor bits, prediction rows, cu_rows and tile ranges, bit-exact."""
import numpy as np
import pytest
import torch

import synthetic as SY
from oracle import tree as OT
from tests.gpu_cases import expected_tile_meta, packed, step_for

pytestmark = pytest.mark.gpu

SMALL = [
    dict(trees=[(300, 40, 9)], W=4),
    dict(trees=[(300, 40, 9)], W=4, pack_terminal=False),
    dict(trees=[(129, 0, 5), (77, 70, 3), (512, 100, 17)], W=3),           # ragged multi-tree
    dict(trees=[(200, 10, 6)], W=1, anchors=[10, 199, 199, 50, 10, 120]),  # W=1, a_b=P, a_b=T-1, duplicates
    dict(trees=[(200, 10, 6)], W=1, pack_terminal=False, anchors=[10, 199, 199, 50, 10, 120]),
    dict(trees=[(90, 5, 4)], W=64, anchors=[60, 5, 89, 30]),                 # full-width ancestor bits, unsorted
    dict(trees=[(64, 8, 0), (10, 2, 3)], W=5),                               # a tree without branches
]


def run_mask(case):
    st = step_for(case, with_grad=False)
    st.build_mask()
    torch.cuda.synchronize()
    return st


def compare_rows(st, case, pt, rows):
    f = OT.compact_fields(pt, rows)
    rows = np.asarray(rows)
    assert np.array_equal(st.pos.cpu().numpy()[rows], f["pos"])
    assert np.array_equal(st.trunk_limit.cpu().numpy()[rows], f["trunk_limit"])
    assert np.array_equal(st.branch_of.cpu().numpy()[rows], f["branch_of"])
    assert np.array_equal(st.anc_bits.cpu().numpy().view(np.uint64)[rows], f["anc_bits"])


@pytest.mark.parametrize("spec", SMALL, ids=range(len(SMALL)))
def test_mask_bit_exact_small(spec):
    spec = dict(spec)
    case = SY.make_case("mask", spec.pop("trees"), Hq=2, Hkv=1, d=32, dtype="bf16", vocab=0, seed=3, **spec)
    st = run_mask(case)
    pt = packed(case)
    assert st.check_status() == 0
    compare_rows(st, case, pt, range(pt.num_rows))
    assert np.array_equal(st.pred_rows.cpu().numpy()[:st.R], OT.prediction_rows(pt))
    assert np.array_equal(st.cu_rows.cpu().numpy(), pt.cu_rows)
    meta = st.tile_meta.cpu().numpy()[:st.num_tiles]
    assert np.array_equal(meta, expected_tile_meta(pt, OT.compact_fields(pt)))


@pytest.mark.parametrize("wl", [2, 3, 4, 5])
def test_mask_bit_exact_full_size_sampled(wl):
    case = SY.make_workload(wl, with_logits=False)
    st = run_mask(case)
    pt = packed(case)
    assert st.check_status() == 0
    rng = np.random.default_rng(wl)
    N = pt.num_rows
    rows = sorted(set(rng.choice(N, size=64, replace=False).tolist()) | {0, N - 1, int(pt.cu_rows[1]) - 1})
    compare_rows(st, case, pt, rows)
    assert np.array_equal(st.pred_rows.cpu().numpy()[:st.R], OT.prediction_rows(pt))
    # invariants that hold at any size
    pos = st.pos.cpu().numpy()
    tl = st.trunk_limit.cpu().numpy()
    bits = st.anc_bits.cpu().numpy().view(np.uint64)
    trunk = st.branch_of.cpu().numpy() < 0
    assert np.all((pos == tl)[trunk]) and np.all(bits[trunk] == 0)
    i = pos - tl
    assert np.all(bits[~trunk] == (np.uint64(1) << i[~trunk].astype(np.uint64)) - np.uint64(1))


def test_anchor_out_of_range_sets_flag():
    case = SY.make_case("bad", [(100, 20, 3)], W=2, Hq=2, Hkv=1, d=32, dtype="bf16", vocab=0,
                        anchors=[25, 5, 40])
    st = step_for(case, with_grad=False)
    st.build_mask()
    torch.cuda.synchronize()
    assert st.check_status() & 1
    # the clamped anchor keeps every field inside the tree
    tl = st.trunk_limit.cpu().numpy()
    assert tl.max() <= 99 and tl.min() >= 0
