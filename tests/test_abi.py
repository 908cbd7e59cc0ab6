"""The C ABI library loads, exports every symbol include/specopd.h declares,
and its host-side logic (counts, argument validation) is right.  No kernel is
launched: everything here runs without a GPU."""
import ctypes
import os
import re

import numpy as np
import pytest

from oracle import tree as T

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "specopd.h")


@pytest.fixture(scope="module")
def S():
    from tree_attention_masked_b200.build import build
    build()
    from tree_attention_masked_b200 import specopd
    return specopd


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*(specopd_[a-z_0-9]+)\s*\(", text, flags=re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ["specopd_build_tree_mask", "specopd_tree_attention", "specopd_tv_overlap", "specopd_e2e_tv_loss",
              "specopd_tv_overlap_e2e", "specopd_rope"]:
        assert n in names


def test_library_exports_every_declared_symbol(S):
    lib = ctypes.CDLL(S.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert sorted(S.EXPORTED) == declared_functions()


CASES = [
    ([12], [3], [4], [3, 7, 11, 5], 3, True),
    ([12], [3], [4], [3, 7, 11, 5], 3, False),
    ([300, 129, 1], [10, 0, 0], [7, 2, 0], [10, 299, 50, 60, 70, 80, 90, 5, 128], 5, True),
    ([10], [4], [5], [4, 9, 6, 5, 8], 1, False),
]


@pytest.mark.parametrize("trunk,prompt,nb,anc,W,ptf", CASES)
def test_counts_match_oracle(S, trunk, prompt, nb, anc, W, ptf):
    import torch
    trees = S.Trees(trunk, prompt, nb, W, torch.zeros(0, dtype=torch.int32), ptf)
    pt = T.pack(trunk, prompt, nb, anc, W, ptf)
    assert S.specopd_tree_packed_rows(trees) == pt.num_rows
    assert S.specopd_tree_num_predictions(trees) == len(T.prediction_rows(pt))
    tiles = sum((int(pt.cu_rows[t + 1] - pt.cu_rows[t]) + 127) // 128 for t in range(len(trunk)))
    assert S.specopd_tree_num_tiles(trees) == tiles


@pytest.mark.parametrize("trunk,prompt,nb,W", [
    ([12], [12], [1], 2),     # prompt covers the whole trunk: no reference position
    ([0], [0], [0], 2),       # empty trunk
    ([12], [3], [-1], 2),
    ([12], [3], [1], 0),
    ([12], [3], [1], 65),
])
def test_bad_descriptions_rejected(S, trunk, prompt, nb, W):
    import torch
    trees = S.Trees(trunk, prompt, nb, W, torch.zeros(0, dtype=torch.int32))
    with pytest.raises(S.SpecopdError):
        S.specopd_tree_packed_rows(trees)


def test_too_many_trees_rejected(S):
    import torch
    n = S.MAX_TREES + 1
    trees = S.Trees([4] * n, [0] * n, [0] * n, 2, torch.zeros(0, dtype=torch.int32))
    with pytest.raises(S.SpecopdError):
        S.specopd_tree_packed_rows(trees)


def test_argument_errors_before_launch(S):
    lib = S._c
    # null logits with rows > 0, misaligned leading dimension, unknown dtype
    assert lib["specopd_tv_overlap"](None, None, 1, 4, 10, 10, 10, None, None, None, None, None, None) == -1
    assert lib["specopd_tv_overlap"](16, 16, 1, 4, 10, 12, 12, 16, None, None, None, 16, None) == -6
    assert lib["specopd_tv_overlap"](16, 16, 7, 4, 10, 16, 16, 16, None, None, None, 16, None) == -3
    # rows must be num_branches * W for the fused entry point
    assert lib["specopd_tv_overlap_e2e"](16, 16, 1, 5, 8, 8, 8, 2, 2, 0.0, 16, 16, None, 0, 256, 1 << 20, 16,
                                         None) == -2
    # workspace too small
    need = S.specopd_overlap_workspace_bytes(4, 8, 2)
    assert lib["specopd_tv_overlap_e2e"](16, 16, 1, 4, 8, 8, 8, 2, 2, 0.0, 16, 16, None, 0, 256, need - 1, 16,
                                         None) == -5
    # attention: head count not a multiple of KV heads, d outside the range
    assert lib["specopd_tree_attention"](16, 16, 16, 16, 1, 8, 3, 2, 128, 1e4, 0.0, 16, 16, 16, 16, 1, 256, 1 << 20,
                                         16, None) == -2
    assert lib["specopd_tree_attention"](16, 16, 16, 16, 1, 8, 4, 2, 48, 1e4, 0.0, 16, 16, 16, 16, 1, 256, 1 << 20,
                                         16, None) == -2
    assert lib["specopd_rope"](16, 16, 16, 16, 1, 4, 2, 2, 6, 16, 1e4, None) == -2
    # one of Hq / Hkv may be 0 (that tensor is skipped and may be null), not both
    assert lib["specopd_rope"](16, 16, 16, 16, 1, 4, 0, 0, 8, 16, 1e4, None) == -2
    assert lib["specopd_rope"](None, 16, None, 16, 1, 0, 0, 2, 8, 16, 1e4, None) == 0   # N = 0: nothing enqueued
    assert lib["specopd_rope"](None, 16, None, 16, 1, 4, 0, 2, 8, None, 1e4, None) == -1  # pos required
    assert lib["specopd_rope"](None, 16, None, 16, 1, 4, 2, 2, 8, 16, 1e4, None) == -1    # q needed when Hq > 0
    # attention on a run of tile records: at most one tile per row; none is a no-op
    assert lib["specopd_tree_attention"](16, 16, 16, 16, 1, 8, 4, 2, 128, 0.0, 0.0, 16, 16, 16, 16, 9, None, 0,
                                         16, None) == -2
    assert lib["specopd_tree_attention"](16, 16, 16, 16, 1, 8, 4, 2, 128, 0.0, 0.0, 16, 16, 16, 16, 0, None, 0,
                                         16, None) == 0
    assert lib["specopd_e2e_tv_loss"](16, 2, 0, 0.0, 16, None, None) == -2
    # LM head: hidden sizes must be multiples of 64, rows = num_branches * W,
    # 16-byte aligned operands, a large enough workspace
    lm = lib["specopd_lm_head_overlap"]
    need = S.specopd_lm_head_workspace_bytes(8, 1000)
    assert lm(16, 16, 96, 16, 16, 128, 8, 1000, 2, 4, 0.0, 16, None, None, None, 16, None, None, 0, 256, need, 16, None) == -2
    assert lm(16, 16, 128, 16, 16, 128, 8, 1000, 3, 4, 0.0, 16, None, None, None, 16, None, None, 0, 256, need, 16, None) == -2
    assert lm(24, 16, 128, 16, 16, 128, 8, 1000, 2, 4, 0.0, 16, None, None, None, 16, None, None, 0, 256, need, 16, None) == -6
    assert lm(16, 16, 128, 16, 16, 128, 8, 1000, 2, 4, 0.0, 16, None, None, None, 16, None, None, 0, 256, need - 1,
              16, None) == -5
    assert lm(16, 16, 128, 16, 16, 128, 8, 1000, 2, 4, 0.0, 16, None, None, None, None, None, None, 0, 256, need,
              16, None) == -1
    # a gradient buffer with a leading dimension below V or not a multiple of 4 floats
    assert lm(16, 16, 128, 16, 16, 128, 8, 1000, 2, 4, 0.0, 16, None, None, None, 16, None, 16, 999, 256, need, 16,
              None) == -6
    assert lm(16, 16, 128, 16, 16, 128, 8, 1000, 2, 4, 0.0, 16, None, None, None, 16, None, 16, 1002, 256, need, 16,
              None) == -6
    assert S._c["specopd_status_string"](-5) == b"workspace missing, too small or misaligned"


def test_gdn_argument_errors_before_launch(S):
    import torch
    trees = S.Trees([200], [10], [4], 4, torch.zeros(4, dtype=torch.int32))
    N = S.specopd_tree_packed_rows(trees)
    need = S.specopd_gdn_workspace_bytes(trees, 2)
    # checkpoints after tokens 63, 127, 191; then per trunk chunk (4 of them,
    # the last one partial) and head: W^T, U [128 x 64 each], P [64][64], 64
    # log2 decays, 64 decay ratios and the chunk's decay (padded to 4)
    up = lambda x: (x + 255) // 256 * 256
    assert need == up(3 * 2 * 128 * 128 * 4) + up(4 * 2 * (2 * 64 * 128 + 64 * 64 + 64 + 64 + 4) * 4)
    g = S._c["specopd_gdn_tree"]
    args = lambda **kw: [trees.ref(), kw.get("q", 16), 16, 16, 16, 16, 16, kw.get("N", N), 2, kw.get("dk", 128),
                         kw.get("dv", 128), 256, kw.get("ws", need), 16, None]
    assert g(*args(dk=64)) == -2            # only d_k = d_v = 128
    assert g(*args(dv=96)) == -2
    assert g(*args(N=N - 1)) == -2          # N must be the packed row count
    assert g(*args(q=24)) == -6             # 16-byte alignment
    assert g(*args(ws=need - 1)) == -5      # the checkpoints must fit
    assert g(*args(q=0)) == -1              # null input


def test_sparse_argument_errors_before_launch(S):
    import torch
    trees = S.Trees([200], [10], [4], 4, torch.zeros(4, dtype=torch.int32))
    N = S.specopd_tree_packed_rows(trees)
    tiles = S.specopd_tree_num_tiles(trees)
    need = S.specopd_sparse_workspace_bytes(trees, 4, 2, 32, 8, 4)
    # rotated Q, K; trunk group keys; branch group keys (4 branches x (4 // 8 + 1) slots);
    # chosen groups [N][Hkv][topk]; selection words
    # (the deepest row has (200 + 4) // 8 = 25 complete groups: one word)
    rq, rk, gk, bk = N * 4 * 128 * 2, N * 2 * 128 * 2, (200 // 8) * 2 * 32 * 4, 4 * 1 * 2 * 32 * 4
    lst, words = N * 2 * 4 * 4, N * 2 * 1 * 4
    up = lambda x: (x + 255) // 256 * 256
    assert need == up(rq) + up(rk) + up(gk) + up(bk) + up(lst) + up(words)
    assert S.specopd_sparse_workspace_bytes(trees, 4, 2, 32, 8, 0) == 0
    f = S._c["specopd_sparse_tree_attention"]
    args = lambda **kw: [trees.ref(), kw.get("q", 16), 16, 16, 16, 16, 16, kw.get("N", N), 4, kw.get("Hkv", 2),
                         kw.get("d", 128), 32, kw.get("g", 8), kw.get("topk", 4), 1e4, 0.0, 16,
                         kw.get("tl", 16), 16, 16, kw.get("tiles", tiles), None, 256, kw.get("ws", need), 16, None]
    assert f(*args(d=64)) == -2             # d = 128 only
    assert f(*args(Hkv=3)) == -2            # Hq a multiple of Hkv
    assert f(*args(topk=65)) == -2          # top-k at most 64
    assert f(*args(topk=0)) == -2
    assert f(*args(g=0)) == -2
    assert f(*args(N=N + 1)) == -2
    assert f(*args(tiles=tiles + 1)) == -2  # the mask builder's tile count
    assert f(*args(q=24)) == -6
    assert f(*args(ws=need - 1)) == -5
    assert f(*args(q=0)) == -1
    assert f(*args(tl=0)) == -1             # the mask fields are required
    # more than 1,024 complete groups in one history
    big = S.Trees([3000], [10], [1], 4, torch.zeros(1, dtype=torch.int32))
    nb = S.specopd_tree_packed_rows(big)
    nt = S.specopd_tree_num_tiles(big)
    assert f(big.ref(), 16, 16, 16, 16, 16, 16, nb, 4, 2, 128, 32, 2, 4, 1e4, 0.0, 16, 16, 16, 16, nt, None, 256,
             1 << 30, 16, None) == -2


def test_wait_timeout_diagnostic_argument_errors(S):
    f = S._c["specopd_diag_overlap_wait_timeout"]
    need = S.specopd_overlap_workspace_bytes(8, 100, 2)
    ok = dict(rows=8, V=100, ld=104, nb=2, W=4, grad=16, ldg=100, ws=need)
    args = lambda **kw: [16, 16, kw.get("rows", 8), kw.get("V", 100), kw.get("ld", 104), 104, kw.get("nb", 2),
                         kw.get("W", 4), kw.get("grad", 16), kw.get("ldg", 100), 256, kw.get("ws", need), 16, None]
    assert f(*args(nb=3)) == -2       # rows = num_branches * W
    assert f(*args(nb=0, rows=0)) == -2
    assert f(*args(grad=None)) == -1  # the gradient buffer is required
    assert f(*args(ldg=98)) == -6
    assert f(*args(ld=101)) == -6     # bf16 rows on 16-byte boundaries
    assert f(*args(ws=need - 1)) == -5
    assert ok


def test_static_scratch_size_matches_the_header(S):
    import os
    import re
    hdr = open(os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                            "specopd.h")).read()
    m = re.search(r"#define SPECOPD_STATIC_SCRATCH_BYTES \(\(size_t\)(\d+) << (\d+)\)", hdr)
    assert m, "SPECOPD_STATIC_SCRATCH_BYTES not found"
    assert S.STATIC_SCRATCH_BYTES == int(m.group(1)) << int(m.group(2))


def test_lm_head_shard_and_merge_argument_errors(S):
    f = S._c["specopd_lm_head_shard_phase"]
    need = S.specopd_lm_head_workspace_bytes(8, 512)
    args = lambda **kw: [kw.get("phase", 0), 16, 16, kw.get("Hd", 128), 16, 16, 128, 8, kw.get("V", 512),
                         kw.get("lz2", 16), 16, 16, 16, 16, kw.get("out2", 16), kw.get("ld", 512), 256,
                         kw.get("ws", need), 16, None]
    assert f(*args(phase=3)) == -1          # phases 0, 1, 2
    assert f(*args(Hd=96)) == -2            # hidden sizes in multiples of 64
    assert f(*args(V=0)) == -2
    assert f(*args(phase=0, out2=None)) == -1
    assert f(*args(phase=1, lz2=None)) == -1  # the global normalisers are inputs from phase 1 on
    assert f(*args(phase=2, ld=510)) == -6    # gradient rows: ld >= V_shard, 16-byte aligned
    assert f(*args(ws=need - 1)) == -5
    m = S._c["specopd_merge_parts"]
    assert m(16, 0, 10, 0, 16, None) == -1    # at least one part
    assert m(16, 2, 10, 2, 16, None) == -1    # modes 0 and 1
    assert m(None, 2, 0, 1, None, None) == 0  # nothing to merge


def test_workspace_sizes(S):
    n_tiles = (151936 + 255) // 256
    assert S.specopd_lm_head_workspace_bytes(1024, 151936) >= n_tiles * 1024 * 24 + 3 * 1024 * 4
    assert S.specopd_lm_head_workspace_bytes(-1, 10) == 0
    assert S.specopd_attention_workspace_bytes(S.BF16, 100, 4, 2, 128) == (
        (100 * 4 * 128 * 2 + 255) // 256 * 256 + (100 * 2 * 128 * 2 + 255) // 256 * 256)
    ws = S.specopd_overlap_workspace_bytes(1024, 151936, 64)
    assert ws >= 1024 * 151936 // 8 + 3 * 1024 * 4
