"""Pins for the oracle's RoPE and tree-masked attention (CPU only).

What fixes the answers:
  * packed scoring equals each branch's independent causal scoring
    (daiwk.github.io write-up, section "Inputs and code mapping"); the second
    side runs torch's fp64 scaled_dot_product_attention(is_causal=True) on the
    branch's own sequence at natural positions;
  * rotate-half RoPE is a rotation of each (k, k + d/2) pair by pos * theta^(-2k/d),
    so it preserves norms and makes q.k depend only on the position difference;
  * special cases: one branch at a_b = T-1 is causal attention over T + W tokens;
    Hq = Hkv is plain multi-head attention.
"""
import numpy as np
import pytest

from oracle import attention as A
from oracle import tree as T


def rand_qkv(rng, N, Hq, Hkv, d):
    return (rng.standard_normal((N, Hq, d)), rng.standard_normal((N, Hkv, d)),
            rng.standard_normal((N, Hkv, d)))


CASES = [
    ([24], [6], [5], [6, 10, 23, 10, 15], 4, True, 4, 2, 16),
    ([24], [6], [5], [6, 10, 23, 10, 15], 4, False, 4, 2, 16),
    ([17, 9], [4, 2], [3, 2], [16, 4, 9, 8, 2], 3, True, 6, 3, 8),   # ragged multi-tree, unsorted anchors
    ([11], [0], [4], [0, 3, 10, 3], 1, True, 2, 2, 8),               # W=1, a_b=P=0, duplicate, MHA
    ([8], [2], [1], [7], 6, True, 4, 1, 8),                           # a_b = T-1
]


@pytest.mark.parametrize("trunk,prompt,nb,anc,W,ptf,Hq,Hkv,d", CASES)
def test_tree_attention_equals_independent_causal(trunk, prompt, nb, anc, W, ptf, Hq, Hkv, d):
    pt = T.pack(trunk, prompt, nb, anc, W, ptf)
    rng = np.random.default_rng(11)
    q, k, v = rand_qkv(rng, pt.num_rows, Hq, Hkv, d)
    o_tree = A.tree_attention(pt, q, k, v, theta=1e4)
    o_ind = A.branch_causal_attention(pt, q, k, v, theta=1e4)
    assert np.max(np.abs(o_tree - o_ind)) < 1e-12


def test_single_branch_at_last_anchor_is_plain_causal():
    import torch
    import torch.nn.functional as F
    Tn, W, Hq, d = 10, 5, 2, 8
    pt = T.pack([Tn], [3], [1], [Tn - 1], W)
    rng = np.random.default_rng(5)
    q, k, v = rand_qkv(rng, Tn + W, Hq, Hq, d)
    o = A.tree_attention(pt, q, k, v, theta=1e4)
    pos = np.arange(Tn + W)
    qr, kr = A.rope(q, pos, 1e4), A.rope(k, pos, 1e4)
    ref = F.scaled_dot_product_attention(torch.from_numpy(qr.transpose(1, 0, 2).copy()),
                                         torch.from_numpy(kr.transpose(1, 0, 2).copy()),
                                         torch.from_numpy(v.transpose(1, 0, 2).copy()),
                                         is_causal=True).numpy().transpose(1, 0, 2)
    assert np.max(np.abs(o - ref)) < 1e-12


def test_packed_offsets_instead_of_semantic_positions_is_wrong():
    """Negative control: RoPE at packed offsets breaks the causal equivalence."""
    pt = T.pack([16], [4], [3], [5, 9, 12], 4)
    rng = np.random.default_rng(2)
    q, k, v = rand_qkv(rng, pt.num_rows, 2, 1, 8)
    ind = A.branch_causal_attention(pt, q, k, v, theta=100.0)
    wrong_pos = np.arange(pt.num_rows)
    orig = T.positions
    try:
        T.positions = lambda _pt: wrong_pos
        bad = A.tree_attention(pt, q, k, v, theta=100.0)
    finally:
        T.positions = orig
    assert np.max(np.abs(bad - ind)) > 1e-3


def test_rope_closed_form_d4():
    # d = 4, theta = 1e4: frequencies 1 and 1e-2; element k pairs with k + 2
    x = np.zeros((1, 1, 4))
    x[0, 0, 0] = 1.0
    y = A.rope(x, np.array([3]), 1e4)[0, 0]
    assert np.allclose(y, [np.cos(3.0), 0.0, np.sin(3.0), 0.0], atol=1e-15)
    x = np.zeros((1, 1, 4))
    x[0, 0, 1] = 1.0
    y = A.rope(x, np.array([3]), 1e4)[0, 0]
    assert np.allclose(y, [0.0, np.cos(0.03), 0.0, np.sin(0.03)], atol=1e-15)


def test_rope_is_rotation_and_relative():
    rng = np.random.default_rng(3)
    d = 32
    q = rng.standard_normal((1, 1, d))
    k = rng.standard_normal((1, 1, d))
    for p in [0, 5, 1234]:
        assert abs(np.linalg.norm(A.rope(q, np.array([p]), 1e4)) - np.linalg.norm(q)) < 1e-12
    dots = []
    for shift in [0, 7, 300]:
        qa = A.rope(q, np.array([40 + shift]), 1e4)
        ka = A.rope(k, np.array([25 + shift]), 1e4)
        dots.append(float((qa * ka).sum()))
    assert max(dots) - min(dots) < 1e-10
    assert np.allclose(A.rope(q, np.array([0]), 1e4), q)


def test_gqa_head_map():
    """Query head h reads KV head h // (Hq/Hkv): duplicating KV heads gives MHA."""
    pt = T.pack([9], [2], [2], [3, 8], 3)
    rng = np.random.default_rng(4)
    q, k, v = rand_qkv(rng, pt.num_rows, 6, 2, 8)
    o_gqa = A.tree_attention(pt, q, k, v, theta=1e4)
    o_mha = A.tree_attention(pt, q, np.repeat(k, 3, axis=1), np.repeat(v, 3, axis=1), theta=1e4)
    assert np.max(np.abs(o_gqa - o_mha)) < 1e-14
