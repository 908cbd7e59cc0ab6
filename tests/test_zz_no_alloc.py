"""The allocation-free overlap entry point against the regular one.

specopd_tv_overlap_e2e_static serves callers that cannot hand the library a
device workspace (their memory belongs to another allocator, or their hot loop
must not call cudaMalloc/cudaFree, which can stall the device).  It runs the
same fused overlap / E2E-TV / gradient pass with the library's own fixed
scratch array.  This file checks, through the C ABI, that two calls in a row
give the regular entry point's results, and that a batch too large for the
fixed scratch is refused before anything runs.
"""
import numpy as np
import pytest
import torch

import synthetic as SY
from tests.gpu_cases import step_for


def _lib():
    from tree_attention_masked_b200.build import build
    build()
    from tree_attention_masked_b200 import specopd
    return specopd


def test_too_large_batch_is_refused():
    S = _lib()
    rows, V, nb = 4096, 151936, 256
    assert S.specopd_overlap_workspace_bytes(rows, V, nb) > S.STATIC_SCRATCH_BYTES
    rc = S._c["specopd_tv_overlap_e2e_static"](16, 16, S.BF16, rows, V, V, V, nb, 16, 0.0, 16, 16, 16, V, 16, None)
    assert rc == -5  # SPECOPD_ERR_WORKSPACE: nothing was enqueued


@pytest.mark.gpu
@pytest.mark.parametrize("dtype,B,W,V", [("bf16", 4, 16, 151936), ("f32", 3, 5, 4099)])
def test_static_scratch_matches_workspace_entry_point(dtype, B, W, V):
    S = _lib()
    case = SY.make_case("noalloc", [(B + 8, 2, B)], W=W, Hq=1, Hkv=1, d=32, dtype=dtype, vocab=V, sig_t=3.0,
                        sig_n=1.5, seed=21, inactive_frac=0.02)
    st = step_for(case)
    assert S.specopd_overlap_workspace_bytes(st.R, V, st.num_branches) <= S.STATIC_SCRATCH_BYTES
    st.overlap()
    torch.cuda.synchronize()
    assert st.check_status() == 0
    ref_alpha = st.alpha[:st.R].double().cpu().numpy()
    ref_loss = float(st.loss.item())
    ref_grad = st.grad.double().cpu().numpy()
    for _ in range(2):  # two calls in a row share, and reuse, the fixed scratch
        alpha = torch.full_like(st.alpha, float("nan"))
        loss = torch.full_like(st.loss, float("nan"))
        # same padded row stride as the regular buffer: rows start on 16-byte boundaries
        grad = torch.full((st.R, st.grad.stride(0)), float("nan"), device="cuda")[:, :V]
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        S.specopd_tv_overlap_e2e_static(st.draft, st.teacher, V, st.num_branches, W, 0.0, alpha, loss, grad, status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        a = alpha[:st.R].double().cpu().numpy()
        g = grad.double().cpu().numpy()
        assert np.max(np.abs(a - ref_alpha)) <= 1e-4
        assert abs(float(loss.item()) - ref_loss) <= 1e-4
        assert np.linalg.norm(g - ref_grad) <= 1e-3 * np.linalg.norm(ref_grad)
