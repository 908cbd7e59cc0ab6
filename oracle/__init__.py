"""fp64 CPU oracle for SpecOPD branch-parallel target scoring.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` use it.  It shares no code with the
CUDA library (no kernels, headers, helpers, tables or constants); the only
common module is ``synthetic``, which draws inputs and holds none of the
method's arithmetic.

Source: "SpecOPD: Branch-Parallel On-Policy Distillation for Speculative
Decoding" as listed on thelatestinai.com (Fig 2, Fig 3, Fig 4, Fig 5, Algorithm 1) and the
daiwk.github.io write-up of it (section "Equations", section "Inputs and code
mapping", section "Checks, negative controls, and limits").

Modules:
  tree       -- proposal-tree packing, parents, visibility, positions,
                prediction rows, and the compact mask encoding derived from them
  attention  -- rotate-half RoPE at semantic positions and tree-masked GQA
                softmax attention, plus the independent per-branch causal form
  overlap    -- full-vocabulary overlap alpha, E2E-TV loss, and the gradient
                with respect to draft logits
  lm_head    -- prediction logits from hidden states and a head, and the
                overlap statistics taken from them
  gdn        -- gated delta rule (GDN linear attention) over a proposal tree,
                every row reading the state of its own history
  sparse     -- sparse attention with branch-consistent indexer groups: top-k
                complete groups per row plus the causal tail
  conv       -- short causal convolution along each row's own history (the
                GDN feature path's convolution that follows branch ancestry)

Every function is plain fp64 NumPy written from the definitions; nothing is
blocked, fused or reordered.
"""
from . import tree, attention, overlap, lm_head, gdn, sparse, conv  # noqa: F401
