"""ctypes binding of libspecopd.so (include/specopd.h).

Argument marshalling only: every function here forwards torch tensors' device
pointers and the current CUDA stream to the C ABI of the same name and raises
if the call returns an error.  All arithmetic runs in the library's kernels.
Importing this module without a built library raises immediately; there is no
fallback path.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libspecopd.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m tree_attention_masked_b200.build`")
_lib = ctypes.CDLL(LIB_PATH)

F32, BF16 = 0, 1
TILE_ROWS = 128
MAX_W = 64
MAX_TREES = 512
FLAG_ANCHOR, FLAG_NONFINITE, FLAG_TIMEOUT = 1, 2, 4

_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_i32 = ctypes.c_int32
_int = ctypes.c_int
_f32 = ctypes.c_float
_f64 = ctypes.c_double
_sz = ctypes.c_size_t


class TreeDesc(ctypes.Structure):
    _fields_ = [("num_trees", _i32), ("W", _i32), ("pack_terminal", _i32),
                ("trunk_len", ctypes.POINTER(_i32)), ("prompt_len", ctypes.POINTER(_i32)),
                ("num_branches", ctypes.POINTER(_i32)), ("anchors", _vp)]


_desc_p = ctypes.POINTER(TreeDesc)


def _sig(name, res, *args):
    f = getattr(_lib, name)
    f.restype = res
    f.argtypes = list(args)
    return f


_c = {
    "specopd_tree_packed_rows": _sig("specopd_tree_packed_rows", _i64, _desc_p),
    "specopd_tree_num_tiles": _sig("specopd_tree_num_tiles", _i64, _desc_p),
    "specopd_tree_num_predictions": _sig("specopd_tree_num_predictions", _i64, _desc_p),
    "specopd_build_tree_mask": _sig("specopd_build_tree_mask", _int, _desc_p, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                    _vp, _vp),
    "specopd_rope": _sig("specopd_rope", _int, _vp, _vp, _vp, _vp, _int, _i64, _int, _int, _int, _vp, _f32, _vp),
    "specopd_attention_workspace_bytes": _sig("specopd_attention_workspace_bytes", _sz, _int, _i64, _int, _int,
                                              _int),
    "specopd_tree_attention": _sig("specopd_tree_attention", _int, _vp, _vp, _vp, _vp, _int, _i64, _int, _int, _int,
                                   _f32, _f32, _vp, _vp, _vp, _vp, _i64, _vp, _sz, _vp, _vp),
    "specopd_overlap_workspace_bytes": _sig("specopd_overlap_workspace_bytes", _sz, _i64, _i64, _i64),
    "specopd_tv_overlap": _sig("specopd_tv_overlap", _int, _vp, _vp, _int, _i64, _i64, _i64, _i64, _vp, _vp, _vp,
                               _vp, _vp, _vp),
    "specopd_e2e_tv_loss": _sig("specopd_e2e_tv_loss", _int, _vp, _i64, _int, _f64, _vp, _vp, _vp),
    "specopd_tv_overlap_e2e": _sig("specopd_tv_overlap_e2e", _int, _vp, _vp, _int, _i64, _i64, _i64, _i64, _i64,
                                   _int, _f64, _vp, _vp, _vp, _i64, _vp, _sz, _vp, _vp),
    "specopd_tv_overlap_e2e_static": _sig("specopd_tv_overlap_e2e_static", _int, _vp, _vp, _int, _i64, _i64,
                                          _i64, _i64, _i64, _int, _f64, _vp, _vp, _vp, _i64, _vp, _vp),
    "specopd_diag_overlap_wait_timeout": _sig("specopd_diag_overlap_wait_timeout", _int, _vp, _vp, _i64, _i64,
                                              _i64, _i64, _i64, _int, _vp, _i64, _vp, _sz, _vp, _vp),
    "specopd_tree_causal_conv": _sig("specopd_tree_causal_conv", _int, _vp, _vp, _int, _i64, _int, _vp, _vp, _int,
                                     _int, _vp, _vp, _vp, _int, _vp),
    "specopd_gdn_workspace_bytes": _sig("specopd_gdn_workspace_bytes", _sz, _desc_p, _int),
    "specopd_gdn_tree": _sig("specopd_gdn_tree", _int, _desc_p, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _int, _int,
                             _int, _vp, _sz, _vp, _vp),
    "specopd_sparse_workspace_bytes": _sig("specopd_sparse_workspace_bytes", _sz, _desc_p, _int, _int, _int, _int,
                                           _int),
    "specopd_sparse_tree_attention": _sig("specopd_sparse_tree_attention", _int, _desc_p, _vp, _vp, _vp, _vp, _vp,
                                          _vp, _i64, _int, _int, _int, _int, _int, _int, _f32, _f32, _vp, _vp, _vp,
                                          _vp, _i64, _vp, _vp, _sz, _vp, _vp),
    "specopd_lm_head_workspace_bytes": _sig("specopd_lm_head_workspace_bytes", _sz, _i64, _i64),
    "specopd_lm_head_overlap": _sig("specopd_lm_head_overlap", _int, _vp, _vp, _int, _vp, _vp, _int, _i64, _i64,
                                    _i64, _int, _f64, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _vp, _sz, _vp, _vp),
    "specopd_lm_head_shard_phase": _sig("specopd_lm_head_shard_phase", _int, _int, _vp, _vp, _int, _vp, _vp, _int,
                                        _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _vp, _sz, _vp, _vp),
    "specopd_merge_parts": _sig("specopd_merge_parts", _int, _vp, _int, _i64, _int, _vp, _vp),
    "specopd_status_string": _sig("specopd_status_string", ctypes.c_char_p, _int),
}

STATIC_SCRATCH_BYTES = 32 << 20

EXPORTED = sorted(_c)


class SpecopdError(RuntimeError):
    pass


def _check(name: str, rc: int) -> None:
    if rc != 0:
        raise SpecopdError(f"{name}: {_c['specopd_status_string'](rc).decode()} ({rc})")


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise SpecopdError(f"unsupported dtype {t.dtype}")


def _contig(*ts):
    for t in ts:
        if t is not None and not t.is_contiguous():
            raise SpecopdError("tensors must be contiguous")


class Trees:
    """A batch of proposal trees: host shape arrays plus the device anchors."""

    def __init__(self, trunk_len: Sequence[int], prompt_len: Sequence[int], num_branches: Sequence[int], W: int,
                 anchors: torch.Tensor, pack_terminal: bool = True):
        n = len(trunk_len)
        self._t = (_i32 * n)(*trunk_len)
        self._p = (_i32 * n)(*prompt_len)
        self._b = (_i32 * n)(*num_branches)
        self.anchors = anchors
        self.desc = TreeDesc(n, W, 1 if pack_terminal else 0, self._t, self._p, self._b,
                             anchors.data_ptr() if anchors.numel() else None)
        self.W = W
        self.num_trees = n

    def ref(self):
        return ctypes.byref(self.desc)


def specopd_tree_packed_rows(trees: Trees) -> int:
    n = _c["specopd_tree_packed_rows"](trees.ref())
    if n < 0:
        _check("specopd_tree_packed_rows", n)
    return n


def specopd_tree_num_tiles(trees: Trees) -> int:
    n = _c["specopd_tree_num_tiles"](trees.ref())
    if n < 0:
        _check("specopd_tree_num_tiles", n)
    return n


def specopd_tree_num_predictions(trees: Trees) -> int:
    n = _c["specopd_tree_num_predictions"](trees.ref())
    if n < 0:
        _check("specopd_tree_num_predictions", n)
    return n


def specopd_build_tree_mask(trees: Trees, pos, trunk_limit, branch_of, anc_bits, pred_rows, cu_rows, tile_meta,
                            status, stream=None) -> None:
    _contig(pos, trunk_limit, branch_of, anc_bits, pred_rows, cu_rows, tile_meta, status)
    _check("specopd_build_tree_mask", _c["specopd_build_tree_mask"](
        trees.ref(), _ptr(pos), _ptr(trunk_limit), _ptr(branch_of), _ptr(anc_bits), _ptr(pred_rows),
        _ptr(cu_rows), _ptr(tile_meta), _ptr(status), _stream(stream)))


def specopd_rope(q, k, q_out, k_out, pos, theta: float, stream=None) -> None:
    """q [N, Hq, d] -> q_out and k [N, Hkv, d] -> k_out; either pair may be None
    (that tensor is skipped)."""
    _contig(q, k, q_out, k_out, pos)
    ref = q if q is not None else k
    N, _, d = ref.shape
    _check("specopd_rope", _c["specopd_rope"](
        _ptr(q), _ptr(k), _ptr(q_out), _ptr(k_out), _dtype(ref), N, 0 if q is None else q.shape[1],
        0 if k is None else k.shape[1], d, _ptr(pos), theta, _stream(stream)))


def specopd_attention_workspace_bytes(dtype: int, N: int, Hq: int, Hkv: int, d: int) -> int:
    return _c["specopd_attention_workspace_bytes"](dtype, N, Hq, Hkv, d)


def specopd_tree_attention(q, k, v, out, pos, trunk_limit, anc_bits, tile_meta, num_tiles: int, rope_theta: float,
                           softmax_scale: float, workspace, status, stream=None) -> None:
    _contig(q, k, v, out, pos, trunk_limit, anc_bits, tile_meta, status)
    N, Hq, d = q.shape
    wb = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("specopd_tree_attention", _c["specopd_tree_attention"](
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _dtype(q), N, Hq, k.shape[1], d, rope_theta, softmax_scale,
        _ptr(pos), _ptr(trunk_limit), _ptr(anc_bits), _ptr(tile_meta), num_tiles, _ptr(workspace), wb,
        _ptr(status), _stream(stream)))


def specopd_overlap_workspace_bytes(rows: int, V: int, num_branches: int) -> int:
    return _c["specopd_overlap_workspace_bytes"](rows, V, num_branches)


def specopd_tv_overlap(draft, teacher, V: int, alpha, q_less, lse_draft, lse_teacher, status, stream=None) -> None:
    _check("specopd_tv_overlap", _c["specopd_tv_overlap"](
        _ptr(draft), _ptr(teacher), _dtype(draft), draft.shape[0], V, draft.stride(0), teacher.stride(0),
        _ptr(alpha), _ptr(q_less), _ptr(lse_draft), _ptr(lse_teacher), _ptr(status), _stream(stream)))


def specopd_e2e_tv_loss(alpha, num_branches: int, W: int, count: float, loss, grad_alpha=None, stream=None) -> None:
    _check("specopd_e2e_tv_loss", _c["specopd_e2e_tv_loss"](
        _ptr(alpha), num_branches, W, count, _ptr(loss), _ptr(grad_alpha), _stream(stream)))


def specopd_tv_overlap_e2e(draft, teacher, V: int, num_branches: int, W: int, count: float, alpha, loss, grad,
                           workspace, status, stream=None) -> None:
    wb = workspace.numel() * workspace.element_size()
    _check("specopd_tv_overlap_e2e", _c["specopd_tv_overlap_e2e"](
        _ptr(draft), _ptr(teacher), _dtype(draft), draft.shape[0], V, draft.stride(0), teacher.stride(0),
        num_branches, W, count, _ptr(alpha), _ptr(loss), _ptr(grad), grad.stride(0) if grad is not None else 0,
        _ptr(workspace), wb, _ptr(status), _stream(stream)))


def specopd_tv_overlap_e2e_static(draft, teacher, V: int, num_branches: int, W: int, count: float, alpha, loss,
                                  grad, status, stream=None) -> None:
    """specopd_tv_overlap_e2e with the library's own fixed scratch instead of a
    caller workspace, for callers that cannot allocate device memory."""
    _check("specopd_tv_overlap_e2e_static", _c["specopd_tv_overlap_e2e_static"](
        _ptr(draft), _ptr(teacher), _dtype(draft), draft.shape[0], V, draft.stride(0), teacher.stride(0),
        num_branches, W, count, _ptr(alpha), _ptr(loss), _ptr(grad), grad.stride(0) if grad is not None else 0,
        _ptr(status), _stream(stream)))


def specopd_lm_head_workspace_bytes(rows: int, V: int) -> int:
    return _c["specopd_lm_head_workspace_bytes"](rows, V)


def specopd_lm_head_overlap(h_draft, head_draft, h_teacher, head_teacher, num_branches: int, W: int,
                            count: float, alpha, loss, workspace, status, q_less=None, lse_draft=None,
                            lse_teacher=None, grad_alpha=None, grad=None, stream=None) -> None:
    """Overlap, E2E-TV loss, dL/dalpha and (with grad) dL/dz from bf16 hidden
    states [rows, H] and heads [V, H] (contiguous); the logits are never stored."""
    _contig(h_draft, head_draft, h_teacher, head_teacher)
    for t in (h_draft, head_draft, h_teacher, head_teacher):
        if t.dtype != torch.bfloat16:
            raise SpecopdError("hidden states and heads must be bf16")
    wb = workspace.numel() * workspace.element_size()
    _check("specopd_lm_head_overlap", _c["specopd_lm_head_overlap"](
        _ptr(h_draft), _ptr(head_draft), h_draft.shape[1], _ptr(h_teacher), _ptr(head_teacher), h_teacher.shape[1],
        h_draft.shape[0], head_draft.shape[0], num_branches, W, count, _ptr(alpha), _ptr(q_less), _ptr(lse_draft),
        _ptr(lse_teacher), _ptr(loss), _ptr(grad_alpha), _ptr(grad), grad.stride(0) if grad is not None else 0,
        _ptr(workspace), wb, _ptr(status), _stream(stream)))


def specopd_gdn_workspace_bytes(trees: Trees, H: int) -> int:
    return _c["specopd_gdn_workspace_bytes"](trees.ref(), H)


def specopd_diag_overlap_wait_timeout(draft, teacher, num_branches: int, W: int, grad, workspace, status,
                                      stream=None) -> None:
    """Failure-detection diagnostic: the fused overlap kernel with no branch
    ever published, so its bounded gradient waits run out (about a second)
    and set FLAG_TIMEOUT in status.  draft, teacher [rows, >= V] bf16 (row
    stride 16-byte aligned), grad [rows, >= V] fp32."""
    wb = workspace.numel() * workspace.element_size()
    _check("specopd_diag_overlap_wait_timeout", _c["specopd_diag_overlap_wait_timeout"](
        _ptr(draft), _ptr(teacher), draft.shape[0], draft.shape[1], draft.stride(0), teacher.stride(0),
        num_branches, W, _ptr(grad), grad.stride(0), _ptr(workspace), wb, _ptr(status), _stream(stream)))


def specopd_tree_causal_conv(x, out, weight, bias, pos, trunk_limit, cu_rows, silu: bool = False,
                             stream=None) -> None:
    """Causal convolution along each row's history: x, out [N, ...] (bf16 or
    fp32, contiguous; the trailing dimensions flattened to C), weight [C, Kw]
    and bias [C] (or None) fp32."""
    _contig(x, out, weight, bias)
    N = x.shape[0]
    C = x.numel() // max(N, 1)
    _check("specopd_tree_causal_conv", _c["specopd_tree_causal_conv"](
        _ptr(x), _ptr(out), _dtype(x), N, C, _ptr(weight), _ptr(bias), weight.shape[1], 1 if silu else 0,
        _ptr(pos), _ptr(trunk_limit), _ptr(cu_rows), cu_rows.shape[0] - 1, _stream(stream)))


def specopd_gdn_tree(trees: Trees, q, k, v, alpha, beta, out, workspace, status, stream=None) -> None:
    """Gated DeltaNet over the packed tree: q, k, v [N, H, 128] bf16, alpha,
    beta [N, H] fp32, out [N, H, 128] fp32 (all contiguous)."""
    _contig(q, k, v, alpha, beta, out)
    wb = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("specopd_gdn_tree", _c["specopd_gdn_tree"](
        trees.ref(), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(out), q.shape[0], q.shape[1],
        q.shape[2], v.shape[2], _ptr(workspace), wb, _ptr(status), _stream(stream)))


def specopd_sparse_workspace_bytes(trees: Trees, Hq: int, Hkv: int, di: int, g: int, topk: int) -> int:
    return _c["specopd_sparse_workspace_bytes"](trees.ref(), Hq, Hkv, di, g, topk)


def specopd_sparse_tree_attention(trees: Trees, q, k, v, qi, ki, out, pos, trunk_limit, anc_bits, tile_meta,
                                  g: int, topk: int, rope_theta: float, workspace, status, selected=None,
                                  softmax_scale: float = 0.0, stream=None) -> None:
    """Sparse attention with branch-consistent indexer groups: q [N, Hq, 128],
    k, v [N, Hkv, 128], qi, ki [N, Hkv, di], out [N, Hq, 128] (bf16, contiguous);
    pos, trunk_limit, anc_bits, tile_meta from specopd_build_tree_mask;
    selected (optional int32 [N, Hkv, topk]) receives the chosen groups."""
    _contig(q, k, v, qi, ki, out, selected)
    wb = workspace.numel() * workspace.element_size()
    _check("specopd_sparse_tree_attention", _c["specopd_sparse_tree_attention"](
        trees.ref(), _ptr(q), _ptr(k), _ptr(v), _ptr(qi), _ptr(ki), _ptr(out), q.shape[0], q.shape[1], k.shape[1],
        q.shape[2], qi.shape[2], g, topk, rope_theta, softmax_scale, _ptr(pos), _ptr(trunk_limit), _ptr(anc_bits),
        _ptr(tile_meta), tile_meta.shape[0], _ptr(selected), _ptr(workspace), wb, _ptr(status), _stream(stream)))


def specopd_lm_head_shard_phase(phase: int, h_draft, head_draft, h_teacher, head_teacher, workspace, status,
                                out1, out2=None, lz2=None, lt2=None, q_less=None, grad_alpha=None,
                                stream=None) -> None:
    """One phase of the LM head + overlap over a vocabulary shard: heads
    [V_shard, H] bf16.  Phase 0: out1/out2 = the shard's base-2 log-sum-exps;
    phase 1 (lz2, lt2 global): out1/out2 = alpha / q_less shares; phase 2
    (lz2, q_less, grad_alpha global): out1 = dL/dz of the shard's columns."""
    _contig(h_draft, head_draft, h_teacher, head_teacher)
    wb = workspace.numel() * workspace.element_size()
    ld = out1.stride(0) if phase == 2 else 0
    _check("specopd_lm_head_shard_phase", _c["specopd_lm_head_shard_phase"](
        phase, _ptr(h_draft), _ptr(head_draft), h_draft.shape[1], _ptr(h_teacher), _ptr(head_teacher),
        h_teacher.shape[1], h_draft.shape[0], head_draft.shape[0], _ptr(lz2), _ptr(lt2), _ptr(q_less),
        _ptr(grad_alpha), _ptr(out1), _ptr(out2), ld, _ptr(workspace), wb, _ptr(status), _stream(stream)))


def specopd_merge_parts(parts, mode: int, out, stream=None) -> None:
    """parts [nparts, n] fp32 -> out [n]: mode 0 sum, mode 1 base-2 log-sum-exp, in part order."""
    _contig(parts, out)
    _check("specopd_merge_parts", _c["specopd_merge_parts"](_ptr(parts), parts.shape[0], parts.shape[1], mode,
                                                            _ptr(out), _stream(stream)))
