"""SpecOPD branch-parallel target scoring on NVIDIA B200 (sm_100a).

The compute path lives in ``libspecopd.so`` (CUDA kernels behind the C ABI
declared in ``include/specopd.h``); ``specopd`` is its ctypes binding and
``scoring.ScoringStep`` runs one full scoring step on device buffers.
Build the library with ``python -m tree_attention_masked_b200.build``.
"""
