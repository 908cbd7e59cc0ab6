"""One SpecOPD target-scoring step on device buffers.

``ScoringStep`` owns the device buffers of one batch of proposal trees and runs
the whole hot path through the C ABI, in order:

  1. specopd_build_tree_mask  -- positions, trunk limits, ancestor bits,
                                 prediction rows, per-tile column ranges
  2. specopd_tree_attention   -- RoPE at semantic positions + tree-masked GQA
                                 attention over every packed row
  3. specopd_tv_overlap_e2e   -- per-prediction overlap alpha, E2E-TV loss and
                                 dL/d(draft logits)

PyTorch only allocates memory and supplies the stream.
"""
from __future__ import annotations

from typing import Optional, Sequence

import torch

from . import specopd as S


class ScoringStep:
    def __init__(self, trunk_len: Sequence[int], prompt_len: Sequence[int], num_branches: Sequence[int], W: int,
                 Hq: int, Hkv: int, d: int, dtype: torch.dtype, vocab: int, device="cuda",
                 pack_terminal: bool = True, theta: float = 1e4, with_grad: bool = True):
        dev = torch.device(device)
        self.device = dev
        self.dtype = dtype
        self.theta = theta
        self.W = W
        self.Hq, self.Hkv, self.d = Hq, Hkv, d
        self.vocab = vocab
        self.with_grad = with_grad
        nb = int(sum(num_branches))
        self.num_branches = nb
        self.anchors = torch.zeros(max(nb, 1), dtype=torch.int32, device=dev)[:nb]
        self.trees = S.Trees(trunk_len, prompt_len, num_branches, W, self.anchors, pack_terminal)
        self.N = S.specopd_tree_packed_rows(self.trees)
        self.num_tiles = S.specopd_tree_num_tiles(self.trees)
        self.R = S.specopd_tree_num_predictions(self.trees)
        N, R = self.N, self.R
        i32 = dict(dtype=torch.int32, device=dev)
        self.q = torch.empty(N, Hq, d, dtype=dtype, device=dev)
        self.k = torch.empty(N, Hkv, d, dtype=dtype, device=dev)
        self.v = torch.empty(N, Hkv, d, dtype=dtype, device=dev)
        self.out = torch.empty(N, Hq, d, dtype=dtype, device=dev)
        self.pos = torch.empty(N, **i32)
        self.trunk_limit = torch.empty(N, **i32)
        self.branch_of = torch.empty(N, **i32)
        self.anc_bits = torch.empty(N, dtype=torch.int64, device=dev)
        self.pred_rows = torch.empty(max(R, 1), **i32)
        self.cu_rows = torch.empty(self.trees.num_trees + 1, **i32)
        self.tile_meta = torch.empty(max(self.num_tiles, 1), 8, **i32)
        self.status = torch.zeros(1, **i32)
        ldt = S.BF16 if dtype == torch.bfloat16 else S.F32
        ws = S.specopd_attention_workspace_bytes(ldt, N, Hq, Hkv, d)
        self.attn_ws = torch.empty(max(ws, 256), dtype=torch.uint8, device=dev)
        # logit rows start on 16-byte boundaries: pad the row stride when needed
        es = torch.tensor([], dtype=dtype).element_size()
        ld = -(-vocab * es // 16) * 16 // es
        ldg = -(-vocab // 4) * 4
        self.draft = torch.empty(R, ld, dtype=dtype, device=dev)[:, :vocab]
        self.teacher = torch.empty(R, ld, dtype=dtype, device=dev)[:, :vocab]
        self.alpha = torch.empty(max(R, 1), dtype=torch.float32, device=dev)
        self.loss = torch.zeros(1, dtype=torch.float32, device=dev)
        self.grad = torch.empty(R, ldg, dtype=torch.float32, device=dev)[:, :vocab] if with_grad else None
        ows = S.specopd_overlap_workspace_bytes(R, vocab, nb)
        self.ov_ws = torch.empty(max(ows, 256), dtype=torch.uint8, device=dev)

    def build_mask(self, stream=None) -> None:
        S.specopd_build_tree_mask(self.trees, self.pos, self.trunk_limit, self.branch_of, self.anc_bits,
                                  self.pred_rows, self.cu_rows, self.tile_meta, self.status, stream)

    def attention(self, stream=None, tiles=None, rows=None) -> None:
        """RoPE + tree attention.  With `tiles` = (t0, t1) only those query
        tiles are scored (rows [r0, r1) = `rows`, the tiles' packed rows): the
        query rows of the range and every key row are rotated into the
        workspace, then the kernel runs on the tiles' records alone."""
        if tiles is None:
            S.specopd_tree_attention(self.q, self.k, self.v, self.out, self.pos, self.trunk_limit, self.anc_bits,
                                     self.tile_meta, self.num_tiles, self.theta, 0.0, self.attn_ws, self.status,
                                     stream)
            return
        t0, t1 = tiles
        if t1 <= t0:
            return
        r0, r1 = rows
        qr, kr = self.rotated()
        S.specopd_rope(self.q[r0:r1], None, qr[r0:r1], None, self.pos[r0:r1], self.theta, stream)
        S.specopd_rope(None, self.k, None, kr, self.pos, self.theta, stream)
        S.specopd_tree_attention(qr, kr, self.v, self.out, self.pos, self.trunk_limit, self.anc_bits,
                                 self.tile_meta[t0:t1], t1 - t0, 0.0, 0.0, None, self.status, stream)

    def rotated(self):
        """Views of the attention workspace holding rotated Q [N, Hq, d] and K [N, Hkv, d]."""
        es = self.q.element_size()
        nq = self.N * self.Hq * self.d
        kq = -(-nq * es // 256) * 256 // es
        flat = self.attn_ws.view(self.q.dtype)
        qr = flat[:nq].view(self.N, self.Hq, self.d)
        kr = flat[kq:kq + self.N * self.Hkv * self.d].view(self.N, self.Hkv, self.d)
        return qr, kr

    def overlap(self, stream=None, count: float = 0.0, branches=None) -> None:
        """Fused overlap / E2E-TV / gradient.  With `branches` = (b0, b1) only
        those branches' rows are scored, normalised by `count` (the whole
        batch's predictions when the branches are split over ranks)."""
        if branches is None:
            S.specopd_tv_overlap_e2e(self.draft, self.teacher, self.vocab, self.num_branches, self.W, count,
                                     self.alpha, self.loss, self.grad, self.ov_ws, self.status, stream)
            return
        b0, b1 = branches
        r0, r1 = b0 * self.W, b1 * self.W
        S.specopd_tv_overlap_e2e(self.draft[r0:r1], self.teacher[r0:r1], self.vocab, b1 - b0, self.W, count,
                                 self.alpha[r0:r1], self.loss, None if self.grad is None else self.grad[r0:r1],
                                 self.ov_ws, self.status, stream)

    def run(self, stream=None) -> None:
        """One pass of the whole hot path (inputs already resident)."""
        self.build_mask(stream)
        self.attention(stream)
        self.overlap(stream)

    def load(self, case, non_blocking: bool = False) -> None:
        """Copy a ``synthetic.Case`` into the device buffers."""
        def dev(x, dt):
            t = torch.from_numpy(x)
            if dt == torch.bfloat16:
                t = t.view(torch.bfloat16)
            return t.to(self.device, non_blocking=non_blocking)
        self.anchors.copy_(torch.from_numpy(case.anchors).to(self.device))
        self.q.copy_(dev(case.q, self.dtype))
        self.k.copy_(dev(case.k, self.dtype))
        self.v.copy_(dev(case.v, self.dtype))
        if case.teacher is not None:
            self.teacher.copy_(dev(case.teacher, self.dtype))
            self.draft.copy_(dev(case.draft, self.dtype))

    def check_status(self) -> int:
        return int(self.status.item())
