"""Failure detection on the GPU without a fault: a bounded in-kernel wait that
runs out sets a status bit, the kernel returns, and the stream stays usable.

The diagnostic entry point runs the fused overlap kernel with every row's
gradient requested but no row's statistics, so no branch is ever published
and every gradient unit's wait (bounded at about a second) gives up.  Nothing
faults, traps or spins without a limit."""
import time

import numpy as np
import pytest
import torch

import synthetic as SY
from tests.gpu_cases import oracle_overlap, step_for
from tree_attention_masked_b200 import specopd as S

pytestmark = pytest.mark.gpu


def test_gradient_wait_runs_out_and_the_stream_stays_usable():
    case = SY.make_case("fd", [(64, 16, 8)], W=4, Hq=2, Hkv=1, d=128, dtype="bf16", vocab=5000, sig_t=3.0,
                        sig_n=1.5, seed=9)
    st = step_for(case)
    torch.cuda.synchronize()
    st.status.zero_()
    t0 = time.perf_counter()
    S.specopd_diag_overlap_wait_timeout(st.draft, st.teacher, st.num_branches, st.W, st.grad, st.ov_ws, st.status)
    torch.cuda.synchronize()
    waited = time.perf_counter() - t0
    assert st.check_status() & S.FLAG_TIMEOUT
    assert waited < 30.0, waited   # the wait is bounded (about a second of GPU clock)
    # the same stream and buffers score correctly afterwards
    st.status.zero_()
    st.overlap()
    torch.cuda.synchronize()
    assert st.check_status() == 0
    alpha = st.alpha.cpu().numpy()[:st.R]
    assert np.max(np.abs(alpha - oracle_overlap(case))) <= 1e-4
