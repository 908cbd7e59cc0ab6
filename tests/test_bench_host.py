"""Host-side accounting of bench.py, checked on the CPU against the oracle.

- visible_pairs (the attention's useful-FLOP count) equals the sum of the
  oracle's visibility sets.
- attention_executed_flops, fed tile records built from the oracle's
  visibility sets, is never below the useful FLOPs, and equals the slot count
  the kernel's work split gives in closed form for one tile and for a pair.
- measured_traffic reports a stored DRAM figure only while the kernel's sources
  hash to the digest stored with it.
- load_peaks reads the measured peaks, else the stated fallback."""
import numpy as np
import pytest

import bench
import synthetic as SY
from oracle import tree as OT

D = 128


def case_for(trees, W, Hq=4, Hkv=2, pack_terminal=True):
    return SY.make_case("b", trees, W=W, Hq=Hq, Hkv=Hkv, d=D, dtype="bf16", vocab=0, seed=5,
                        pack_terminal=pack_terminal)


def tile_meta(case):
    """[row_start, row_end, tree_base, trunk_hi, trunk_full, br_lo, br_hi, 0] per
    128-row tile of each tree, from the oracle's visible columns."""
    pt = OT.pack(case.trunk_len, case.prompt_len, case.num_branches, case.anchors, case.W, case.pack_terminal)
    out = []
    for t in range(len(case.trunk_len)):
        base, end, T = int(pt.cu_rows[t]), int(pt.cu_rows[t + 1]), int(case.trunk_len[t])
        for r0 in range(base, end, 128):
            r1 = min(end, r0 + 128)
            trunk_hi, trunk_full, br_lo, br_hi = base, base + T, None, None
            for r in range(r0, r1):
                vis = OT.visible(pt, r)
                tr = vis[vis < base + T]
                br = vis[vis >= base + T]
                trunk_hi = max(trunk_hi, int(tr.max()) + 1)
                trunk_full = min(trunk_full, int(tr.max()) + 1)
                if br.size:
                    br_lo = int(br.min()) if br_lo is None else min(br_lo, int(br.min()))
                    br_hi = int(br.max()) + 1 if br_hi is None else max(br_hi, int(br.max()) + 1)
            out.append([r0, r1, base, trunk_hi, trunk_full, br_lo or 0, br_hi or 0, 0])
    return np.array(out, dtype=np.int64), pt


@pytest.mark.parametrize("trees,W,ptf", [([(300, 40, 9)], 4, True), ([(129, 0, 5), (77, 70, 3)], 3, True),
                                         ([(200, 10, 6)], 5, False), ([(64, 0, 0)], 1, True)])
def test_visible_pairs_is_the_sum_of_visibility_sets(trees, W, ptf):
    case = case_for(trees, W, pack_terminal=ptf)
    pt = OT.pack(case.trunk_len, case.prompt_len, case.num_branches, case.anchors, case.W, case.pack_terminal)
    assert bench.visible_pairs(case) == sum(len(OT.visible(pt, r)) for r in range(pt.num_rows))


@pytest.mark.parametrize("G", [1, 2, 4, 5])
def test_executed_flops_cover_the_useful_ones(G):
    case = case_for([(700, 100, 12), (260, 30, 5)], 16, Hq=2 * G, Hkv=2)
    meta, _ = tile_meta(case)
    useful = 4.0 * D * case.Hq * bench.visible_pairs(case)
    executed = bench.attention_executed_flops(meta, case.Hkv, G, D)
    assert executed >= useful
    assert executed <= 4.0 * D * case.Hq * sum(int(m[1] - m[0]) * (int(m[3] - m[2]) + int(m[6] - m[5]) + 256)
                                               for m in meta)


def test_executed_flops_closed_forms():
    blk = 4.0 * D * 128 * 128  # one (query head, tile) slot over one 128-column block
    one = np.array([[0, 100, 0, 100, 1, 0, 0, 0]])  # one tile of 100 trunk rows: one block
    assert bench.attention_executed_flops(one, 3, 2, D) == blk * 2 * 3           # two heads per KV head
    assert bench.attention_executed_flops(one, 3, 3, D) == blk * (2 * 3 + 3)     # plus the odd head alone
    two = np.array([[0, 128, 0, 128, 1, 0, 0, 0], [128, 256, 0, 256, 129, 0, 0, 0]])  # one tree, 1 and 2 blocks
    # G = 5: two head pairs per tile (1 and 2 blocks), the odd head on both tiles over the union (2 blocks)
    assert bench.attention_executed_flops(two, 1, 5, D) == blk * (4 * 1 + 4 * 2 + 2 * 2)


def test_traffic_follows_the_sources(monkeypatch):
    digest = bench.source_digest("tree_attention")
    monkeypatch.setitem(bench.MEASURED_TRAFFIC, (9, "tree_attention"), {"bytes": 123.0, "sha": digest, "profile": "-"})
    assert bench.measured_traffic(9, "tree_attention") == 123.0
    monkeypatch.setitem(bench.MEASURED_TRAFFIC, (9, "tree_attention"),
                        {"bytes": 123.0, "sha": "0" * 16, "profile": "-"})
    assert bench.measured_traffic(9, "tree_attention") is None
    assert bench.measured_traffic(8, "tree_attention") is None  # no capture for that workload


def test_peaks(monkeypatch, tmp_path):
    p = bench.load_peaks()
    assert p["hbm"] > 0 and p["bf16"] > 0
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.load_peaks() == dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")
