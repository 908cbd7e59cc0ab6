"""Seeded synthetic inputs for SpecOPD target scoring.

This module only draws random inputs and lays them out in the packed shapes the
scoring path consumes.  It holds none of the method's arithmetic: no masks, no
positions, no attention, no overlap.  Both the fp64 oracle tests and the CUDA
path (tests, bench) take their inputs from here, so the two sides see the same
bytes.

Workloads (SpecOPD: Branch-Parallel On-Policy Distillation for Speculative
Decoding, Fig 2 and Fig 3 for the tree; the 8B GQA and 27B GQA-GDN targets of
the abstract for the attention shapes):

* a proposal tree is a trunk of T tokens (prompt P + reference T-P) followed by
  B branches of W drafted tokens, packed branch by branch;
* anchors are drawn uniformly without replacement from the reference positions
  [P, T-1] (zero-based) and sorted ascending;
* Q/K/V are N(0,1), drawn in fp32 and rounded to bf16 by round-to-nearest-even
  (kept in fp32 for the tiny fp32 case);
* teacher logits t ~ N(0, sigma_t^2); draft logits z = t + N(0, sigma_n^2),
  with the sum formed in fp32 from the stored teacher value and rounded to the
  storage dtype once.

Every tensor draws from its own PCG64 substream
``default_rng([seed, tensor_id, tree_id, chunk])`` so any slice can be
regenerated independently and in parallel.
"""
from __future__ import annotations

import dataclasses
import multiprocessing as mp
from typing import List, Optional, Sequence, Tuple

import numpy as np

# tensor ids of the substreams
_TID_ANCHOR, _TID_Q, _TID_K, _TID_V, _TID_TEACHER, _TID_DRAFT, _TID_MASK, _TID_SHAPE = range(8)
_ROW_CHUNK = 256  # logit rows per substream chunk


def bf16_round(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit pattern (uint16), round to nearest even.  Finite inputs only."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))
    return (rounded >> np.uint32(16)).astype(np.uint16)


def bf16_to_f32(u: np.ndarray) -> np.ndarray:
    """bf16 bit pattern (uint16) -> fp32 (exact)."""
    return (np.ascontiguousarray(u, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def to_f64(x: np.ndarray, dtype: str) -> np.ndarray:
    """Stored tensor -> exact fp64 values."""
    if dtype == "bf16":
        return bf16_to_f32(x).astype(np.float64)
    return np.asarray(x, dtype=np.float32).astype(np.float64)


@dataclasses.dataclass
class Case:
    """One scoring batch: proposal trees plus aligned draft/teacher logits."""
    name: str
    trunk_len: List[int]
    prompt_len: List[int]
    num_branches: List[int]
    W: int
    anchors: np.ndarray          # int32 [sum B], zero-based within each tree, tree-major
    Hq: int
    Hkv: int
    d: int
    dtype: str                   # "bf16" (uint16 storage) or "f32"
    q: np.ndarray                # [N, Hq, d]  pre-RoPE
    k: np.ndarray                # [N, Hkv, d] pre-RoPE
    v: np.ndarray                # [N, Hkv, d]
    vocab: int
    teacher: Optional[np.ndarray]  # [sum B * W, vocab]
    draft: Optional[np.ndarray]    # [sum B * W, vocab]
    theta: float = 1e4
    pack_terminal: bool = True

    @property
    def num_trees(self) -> int:
        return len(self.trunk_len)

    @property
    def rows_per_branch(self) -> int:
        return self.W if self.pack_terminal else self.W - 1

    @property
    def num_rows(self) -> int:
        return int(sum(T + B * self.rows_per_branch for T, B in zip(self.trunk_len, self.num_branches)))

    @property
    def num_predictions(self) -> int:
        return int(sum(self.num_branches)) * self.W


def _draw_anchors(seed: int, tree: int, P: int, T: int, B: int, sort: bool, replace: bool) -> np.ndarray:
    rng = np.random.default_rng([seed, _TID_ANCHOR, tree])
    if replace:
        a = rng.integers(P, T, size=B)
    else:
        if B > T - P:
            raise ValueError(f"cannot draw {B} distinct anchors from {T - P} reference positions")
        a = rng.choice(np.arange(P, T), size=B, replace=False)
    if sort:
        a = np.sort(a)
    return a.astype(np.int32)


def _normal_rows(seed: int, tid: int, tree: int, rows: int, cols: int, sigma: float) -> np.ndarray:
    out = np.empty((rows, cols), dtype=np.float32)
    for c0 in range(0, rows, _ROW_CHUNK):
        c1 = min(rows, c0 + _ROW_CHUNK)
        rng = np.random.default_rng([seed, tid, tree, c0 // _ROW_CHUNK])
        out[c0:c1] = rng.standard_normal((c1 - c0, cols), dtype=np.float32)
    if sigma != 1.0:
        out *= np.float32(sigma)
    return out


def _logit_chunk(args) -> Tuple[int, np.ndarray, np.ndarray]:
    seed, tree, chunk, rows, vocab, sig_t, sig_n, dtype, inactive_frac = args
    rt = np.random.default_rng([seed, _TID_TEACHER, tree, chunk])
    rd = np.random.default_rng([seed, _TID_DRAFT, tree, chunk])
    t32 = rt.standard_normal((rows, vocab), dtype=np.float32)
    t32 *= np.float32(sig_t)
    if dtype == "bf16":
        t_store = bf16_round(t32)
        t32 = bf16_to_f32(t_store)
    else:
        t_store = t32
    n32 = rd.standard_normal((rows, vocab), dtype=np.float32)
    n32 *= np.float32(sig_n)
    z32 = t32 + n32
    if inactive_frac > 0.0:
        rm = np.random.default_rng([seed, _TID_MASK, tree, chunk])
        drop = rm.random((rows, vocab), dtype=np.float32) < np.float32(inactive_frac)
        z32[drop] = np.float32(np.nan)
    if dtype == "bf16":
        z_store = bf16_round(np.nan_to_num(z32, nan=0.0))
        if inactive_frac > 0.0:
            z_store[drop] = np.uint16(0x7FC0)  # bf16 quiet NaN
    else:
        z_store = z32
    return chunk, t_store, z_store


def make_logits(seed: int, rows_per_tree: Sequence[int], vocab: int, sig_t: float, sig_n: float,
                dtype: str, inactive_frac: float = 0.0, workers: int = 0) -> Tuple[np.ndarray, np.ndarray]:
    """Teacher and draft logits [sum rows, vocab], tree-major, rows b-major then i."""
    total = int(sum(rows_per_tree))
    st = np.uint16 if dtype == "bf16" else np.float32
    teacher = np.empty((total, vocab), dtype=st)
    draft = np.empty((total, vocab), dtype=st)
    jobs = []
    base = 0
    offsets = []
    for tree, rows in enumerate(rows_per_tree):
        for c0 in range(0, rows, _ROW_CHUNK):
            r = min(_ROW_CHUNK, rows - c0)
            jobs.append((seed, tree, c0 // _ROW_CHUNK, r, vocab, sig_t, sig_n, dtype, inactive_frac))
            offsets.append(base + c0)
        base += rows
    if workers and len(jobs) > 1:
        ctx = mp.get_context("spawn")
        with ctx.Pool(workers) as pool:
            results = pool.map(_logit_chunk, jobs, chunksize=1)
    else:
        results = [_logit_chunk(j) for j in jobs]
    for off, (_, t, z) in zip(offsets, results):
        teacher[off:off + t.shape[0]] = t
        draft[off:off + z.shape[0]] = z
    return teacher, draft


def make_case(name: str, trees: Sequence[Tuple[int, int, int]], W: int, Hq: int, Hkv: int, d: int,
              dtype: str, vocab: int = 0, sig_t: float = 3.0, sig_n: float = 1.0, seed: int = 0,
              anchors: Optional[Sequence[int]] = None, sort_anchors: bool = True,
              anchor_replace: bool = False, pack_terminal: bool = True, inactive_frac: float = 0.0,
              theta: float = 1e4, workers: int = 0, with_logits: bool = True) -> Case:
    """Build a batch of trees.  ``trees`` lists (T, P, B) per tree.

    ``anchors`` (tree-major, zero-based within each tree) overrides the draw.
    """
    trunk = [int(t[0]) for t in trees]
    prompt = [int(t[1]) for t in trees]
    nb = [int(t[2]) for t in trees]
    if anchors is None:
        parts = [_draw_anchors(seed, i, P, T, B, sort_anchors, anchor_replace)
                 for i, (T, P, B) in enumerate(zip(trunk, prompt, nb))]
        anc = np.concatenate(parts) if parts else np.zeros(0, np.int32)
    else:
        anc = np.asarray(anchors, dtype=np.int32)
    rpb = W if pack_terminal else W - 1
    rows_tree = [T + B * rpb for T, B in zip(trunk, nb)]
    N = int(sum(rows_tree))
    qs, ks, vs = [], [], []
    for i, n in enumerate(rows_tree):
        qs.append(_normal_rows(seed, _TID_Q, i, n, Hq * d, 1.0))
        ks.append(_normal_rows(seed, _TID_K, i, n, Hkv * d, 1.0))
        vs.append(_normal_rows(seed, _TID_V, i, n, Hkv * d, 1.0))
    cat = lambda xs, c: (np.concatenate(xs) if xs else np.zeros((0, c), np.float32))
    q = cat(qs, Hq * d).reshape(N, Hq, d)
    k = cat(ks, Hkv * d).reshape(N, Hkv, d)
    v = cat(vs, Hkv * d).reshape(N, Hkv, d)
    if dtype == "bf16":
        q, k, v = bf16_round(q), bf16_round(k), bf16_round(v)
    elif dtype != "f32":
        raise ValueError(dtype)
    teacher = draft = None
    if with_logits and vocab > 0:
        teacher, draft = make_logits(seed, [B * W for B in nb], vocab, sig_t, sig_n, dtype,
                                     inactive_frac, workers)
    return Case(name, trunk, prompt, nb, W, anc, Hq, Hkv, d, dtype, q, k, v, vocab, teacher, draft,
                theta, pack_terminal)


# ---------------------------------------------------------------------------
# The five workloads: tiny fp32 tree, 8B-style GQA tree, 8 ragged trees,
# 16K agentic-style trunk, 27B-scale 32K trunk with a 248K vocabulary.
# ---------------------------------------------------------------------------

WORKLOADS = {
    1: "tiny-fp32: 1 tree T=64 (P=16), B=4 W=4, 4/2 heads d=64, fp32, V=512",
    2: "gqa8b: 1 tree T=4096 (P=1024), B=64 W=16, 32/8 heads d=128, bf16, V=151936",
    3: "ragged8: 8 trees T~U[1024,4096] (P=T/4), B~U[16,64], W=8, 32/8 heads d=128, bf16, V=151936",
    4: "long16k: 1 tree T=16384 (P=4096), B=256 W=16, 32/8 heads d=128, bf16, V=151936",
    5: "scale27b: 1 tree T=32768 (P=8192), B=512 W=16, 40/8 heads d=128, bf16, V=248320",
}


def ragged_tree_shapes(seed: int = 0, trees: int = 8) -> List[Tuple[int, int, int]]:
    rng = np.random.default_rng([seed, _TID_SHAPE, 0])
    T = rng.integers(1024, 4097, size=trees)
    B = rng.integers(16, 65, size=trees)
    return [(int(t), int(t) // 4, int(b)) for t, b in zip(T, B)]


def make_workload(i: int, seed: int = 0, workers: int = 0, with_logits: bool = True) -> Case:
    if i == 1:
        return make_case("tiny-fp32", [(64, 16, 4)], W=4, Hq=4, Hkv=2, d=64, dtype="f32", vocab=512,
                         sig_t=3.0, sig_n=1.0, seed=seed, workers=workers, with_logits=with_logits)
    if i == 2:
        return make_case("gqa8b", [(4096, 1024, 64)], W=16, Hq=32, Hkv=8, d=128, dtype="bf16",
                         vocab=151936, sig_t=3.0, sig_n=1.5, seed=seed, workers=workers,
                         with_logits=with_logits)
    if i == 3:
        return make_case("ragged8", ragged_tree_shapes(seed), W=8, Hq=32, Hkv=8, d=128, dtype="bf16",
                         vocab=151936, sig_t=3.0, sig_n=1.5, seed=seed, workers=workers,
                         with_logits=with_logits)
    if i == 4:
        return make_case("long16k", [(16384, 4096, 256)], W=16, Hq=32, Hkv=8, d=128, dtype="bf16",
                         vocab=151936, sig_t=3.0, sig_n=0.5, seed=seed, workers=workers,
                         with_logits=with_logits)
    if i == 5:
        return make_case("scale27b", [(32768, 8192, 512)], W=16, Hq=40, Hkv=8, d=128, dtype="bf16",
                         vocab=248320, sig_t=4.0, sig_n=2.0, seed=seed, workers=workers,
                         with_logits=with_logits)
    raise ValueError(f"unknown workload {i}")


# ---------------------------------------------------------------------------
# Hidden states and LM heads (prediction logits formed from them, never stored)
# ---------------------------------------------------------------------------

_TID_H_TEACHER, _TID_W_TEACHER, _TID_H_DRAFT, _TID_W_DRAFT = range(100, 104)


@dataclasses.dataclass
class LmHeadCase:
    name: str
    num_branches: int
    W: int
    V: int
    Hd: int
    Ht: int
    h_draft: np.ndarray   # [rows, Hd] bf16 bits (uint16)
    w_draft: np.ndarray   # [V, Hd]
    h_teacher: np.ndarray  # [rows, Ht]
    w_teacher: np.ndarray  # [V, Ht]

    @property
    def rows(self) -> int:
        return self.num_branches * self.W


def _head_chunk(args) -> Tuple[int, np.ndarray, np.ndarray]:
    """Rows [256 c, 256 c + 256) of both heads (the substreams of _normal_rows)."""
    seed, c, rows, Hd, Ht, sig_t, sig_n = args
    rt = np.random.default_rng([seed, _TID_W_TEACHER, 0, c])
    wt = rt.standard_normal((rows, Ht), dtype=np.float32) * np.float32(sig_t / np.sqrt(Ht))
    wt_b = bf16_round(wt)
    rd = np.random.default_rng([seed, _TID_W_DRAFT, 0, c])
    if Hd == Ht:
        noise = rd.standard_normal((rows, Hd), dtype=np.float32) * np.float32(sig_n / np.sqrt(Hd))
        wd_b = bf16_round(bf16_to_f32(wt_b) + noise)
    else:
        wd_b = bf16_round(rd.standard_normal((rows, Hd), dtype=np.float32) * np.float32(sig_t / np.sqrt(Hd)))
    return c, wd_b, wt_b


def make_lm_head_case(name: str, num_branches: int, W: int, V: int, Hd: int, Ht: int, sig_t: float,
                      sig_n: float, seed: int = 0, workers: int = 0) -> LmHeadCase:
    """Teacher hidden states h_t ~ N(0, 1) and head w_t ~ N(0, sig_t^2 / Ht), so
    that teacher logits have standard deviation about sig_t.  With Hd == Ht the
    draft reads the same hidden states through w_d = w_t + N(0, sig_n^2 / Hd)
    (its logits are the teacher's plus noise of deviation about sig_n);
    otherwise it has its own h_d ~ N(0, 1) and w_d ~ N(0, sig_t^2 / Hd).
    Everything is drawn in fp32 and rounded to bf16 once; the heads are drawn
    in 256-row chunks, each from its own substream, so `workers` processes
    give the same bytes as one."""
    rows = num_branches * W
    ht = _normal_rows(seed, _TID_H_TEACHER, 0, rows, Ht, 1.0)
    jobs = [(seed, c, min(_ROW_CHUNK, V - c * _ROW_CHUNK), Hd, Ht, sig_t, sig_n)
            for c in range((V + _ROW_CHUNK - 1) // _ROW_CHUNK)]
    if workers and len(jobs) > 1:
        with mp.get_context("spawn").Pool(workers) as pool:
            results = pool.map(_head_chunk, jobs, chunksize=4)
    else:
        results = [_head_chunk(j) for j in jobs]
    wd_b = np.empty((V, Hd), dtype=np.uint16)
    wt_b = np.empty((V, Ht), dtype=np.uint16)
    for c, d, t in results:
        wd_b[c * _ROW_CHUNK:c * _ROW_CHUNK + d.shape[0]] = d
        wt_b[c * _ROW_CHUNK:c * _ROW_CHUNK + t.shape[0]] = t
    hd_b = bf16_round(ht) if Hd == Ht else bf16_round(_normal_rows(seed, _TID_H_DRAFT, 0, rows, Hd, 1.0))
    return LmHeadCase(name, num_branches, W, V, Hd, Ht, hd_b, wd_b, bf16_round(ht), wt_b)


# ---------------------------------------------------------------------------
# Gated DeltaNet features per packed row (consumed as given by the GDN path)
# ---------------------------------------------------------------------------

_TID_GDN_Q, _TID_GDN_K, _TID_GDN_V, _TID_GDN_A, _TID_GDN_B = range(110, 115)


@dataclasses.dataclass
class GdnCase:
    name: str
    trunk_len: List[int]
    prompt_len: List[int]
    num_branches: List[int]
    W: int
    H: int
    pack_terminal: bool
    anchors: np.ndarray   # int32 [sum B], zero-based within each tree
    q: np.ndarray         # [N, H, 128] bf16 bits
    k: np.ndarray         # [N, H, 128] bf16 bits, rows of unit norm before rounding
    v: np.ndarray         # [N, H, 128] bf16 bits
    alpha: np.ndarray     # [N, H] fp32 in [0.9, 1)
    beta: np.ndarray      # [N, H] fp32 in [0.1, 0.9)

    @property
    def num_rows(self) -> int:
        return self.q.shape[0]


def make_gdn_case(name: str, trees: Sequence[Tuple[int, int, int]], W: int, H: int, seed: int = 0,
                  pack_terminal: bool = True, anchors: Sequence[Sequence[int]] = None) -> GdnCase:
    """Per packed row and head: q ~ N(0, 1/128), k = a N(0, I) draw scaled to
    unit norm, v ~ N(0, 1) (all rounded to bf16 once), decay alpha ~ U[0.9, 1)
    and write strength beta ~ U[0.1, 0.9) in fp32.  Anchors as for the
    attention workloads unless given per tree."""
    d = 128
    rpb = W if pack_terminal else W - 1
    N = int(sum(T + B * rpb for T, _, B in trees))
    anc = []
    for t, (T, P, B) in enumerate(trees):
        anc.append(np.asarray(anchors[t], dtype=np.int32) if anchors is not None
                   else _draw_anchors(seed, t, P, T, B, True, False))
    q = _normal_rows(seed, _TID_GDN_Q, 0, N, H * d, 1.0 / np.sqrt(d)).reshape(N, H, d)
    k = _normal_rows(seed, _TID_GDN_K, 0, N, H * d, 1.0).reshape(N, H, d)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = _normal_rows(seed, _TID_GDN_V, 0, N, H * d, 1.0).reshape(N, H, d)
    rng_a = np.random.default_rng([seed, _TID_GDN_A, 0, 0])
    rng_b = np.random.default_rng([seed, _TID_GDN_B, 0, 0])
    alpha = rng_a.uniform(0.9, 1.0, size=(N, H)).astype(np.float32)
    beta = rng_b.uniform(0.1, 0.9, size=(N, H)).astype(np.float32)
    return GdnCase(name, [t[0] for t in trees], [t[1] for t in trees], [t[2] for t in trees], W, H, pack_terminal,
                   np.concatenate(anc) if anc else np.zeros(0, np.int32), bf16_round(q), bf16_round(k),
                   bf16_round(v), alpha, beta)


# ---------------------------------------------------------------------------
# Sparse attention with indexer groups: attention and indexer features per row
# ---------------------------------------------------------------------------

_TID_SP_Q, _TID_SP_K, _TID_SP_V, _TID_SP_QI, _TID_SP_KI = range(120, 125)


@dataclasses.dataclass
class SparseCase:
    name: str
    trunk_len: List[int]
    prompt_len: List[int]
    num_branches: List[int]
    W: int
    Hq: int
    Hkv: int
    di: int
    pack_terminal: bool
    anchors: np.ndarray   # int32 [sum B]
    q: np.ndarray         # [N, Hq, 128] bf16 bits
    k: np.ndarray         # [N, Hkv, 128]
    v: np.ndarray         # [N, Hkv, 128]
    qi: np.ndarray        # [N, Hkv, di] indexer queries
    ki: np.ndarray        # [N, Hkv, di] indexer keys

    @property
    def num_rows(self) -> int:
        return self.q.shape[0]


def make_sparse_case(name: str, trees: Sequence[Tuple[int, int, int]], W: int, Hq: int, Hkv: int, di: int,
                     seed: int = 0, pack_terminal: bool = True) -> SparseCase:
    """Attention features q, k, v ~ N(0, 1) and indexer features qi, ki ~ N(0, 1),
    drawn in fp32 and rounded to bf16 once; anchors as for the attention workloads."""
    d = 128
    rpb = W if pack_terminal else W - 1
    N = int(sum(T + B * rpb for T, _, B in trees))
    anc = [_draw_anchors(seed, t, P, T, B, True, False) for t, (T, P, B) in enumerate(trees)]
    f = lambda tid, heads, width: bf16_round(_normal_rows(seed, tid, 0, N, heads * width, 1.0)).reshape(N, heads, width)
    return SparseCase(name, [t[0] for t in trees], [t[1] for t in trees], [t[2] for t in trees], W, Hq, Hkv, di,
                      pack_terminal, np.concatenate(anc) if anc else np.zeros(0, np.int32),
                      f(_TID_SP_Q, Hq, d), f(_TID_SP_K, Hkv, d), f(_TID_SP_V, Hkv, d), f(_TID_SP_QI, Hkv, di),
                      f(_TID_SP_KI, Hkv, di))


_TID_CV_X, _TID_CV_W, _TID_CV_B = range(130, 133)


@dataclasses.dataclass
class ConvCase:
    """Features of the packed rows of some trees and a depthwise filter."""
    name: str
    trunk_len: List[int]
    prompt_len: List[int]
    num_branches: List[int]
    W: int
    pack_terminal: bool
    anchors: np.ndarray   # int32 [sum B]
    dtype: str            # "bf16" (uint16 storage) or "f32"
    x: np.ndarray         # [N, C]
    weight: np.ndarray    # [C, Kw] fp32
    bias: np.ndarray      # [C] fp32

    @property
    def num_rows(self) -> int:
        return self.x.shape[0]


def make_conv_case(name: str, trees: Sequence[Tuple[int, int, int]], W: int, C: int, Kw: int, dtype: str = "bf16",
                   seed: int = 0, pack_terminal: bool = True) -> ConvCase:
    """Features x ~ N(0, 1) (drawn in fp32, rounded to bf16 once for bf16),
    filter weights ~ N(0, 1/Kw) and bias ~ N(0, 0.1^2) in fp32; anchors as for
    the attention workloads."""
    rpb = W if pack_terminal else W - 1
    N = int(sum(T + B * rpb for T, _, B in trees))
    anc = [_draw_anchors(seed, t, P, T, B, True, False) for t, (T, P, B) in enumerate(trees)]
    x = _normal_rows(seed, _TID_CV_X, 0, N, C, 1.0)
    if dtype == "bf16":
        x = bf16_round(x)
    w = np.random.default_rng([seed, _TID_CV_W, 0, 0]).normal(0.0, 1.0 / np.sqrt(Kw), size=(C, Kw))
    b = np.random.default_rng([seed, _TID_CV_B, 0, 0]).normal(0.0, 0.1, size=C)
    return ConvCase(name, [t[0] for t in trees], [t[1] for t in trees], [t[2] for t in trees], W, pack_terminal,
                    np.concatenate(anc) if anc else np.zeros(0, np.int32), dtype, x,
                    w.astype(np.float32), b.astype(np.float32))
