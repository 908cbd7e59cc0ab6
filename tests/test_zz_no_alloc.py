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


def test_argument_errors_come_before_the_size_check():
    """A bad call reports its own error, even when its shape is too large for
    the fixed scratch."""
    S = _lib()
    f = S._c["specopd_tv_overlap_e2e_static"]
    rows, V, nb = 4096, 151936, 256
    assert f(16, 16, 7, rows, V, V, V, nb, 16, 0.0, 16, 16, 16, V, 16, None) == -3          # dtype
    assert f(16, 16, S.BF16, rows, V, V, V, nb + 1, 16, 0.0, 16, 16, 16, V, 16, None) == -2  # rows != nb W
    assert f(16, 16, S.BF16, rows, V, V, V, nb, 16, 0.0, 16, None, 16, V, 16, None) == -1    # loss
    assert f(16, 24, S.BF16, rows, V, V, V, nb, 16, 0.0, 16, 16, 16, V, 16, None) == -6      # alignment


def _case(dtype, B, W, V, seed):
    case = SY.make_case("noalloc", [(B + 8, 2, B)], W=W, Hq=1, Hkv=1, d=32, dtype=dtype, vocab=V, sig_t=3.0,
                        sig_n=1.5, seed=seed, inactive_frac=0.02)
    st = step_for(case)
    st.overlap()
    torch.cuda.synchronize()
    assert st.check_status() == 0
    return st, (st.alpha[:st.R].double().cpu().numpy(), float(st.loss.item()), st.grad.double().cpu().numpy())


def _static_call(S, st, V, W, ref):
    alpha = torch.full_like(st.alpha, float("nan"))
    loss = torch.full_like(st.loss, float("nan"))
    # same padded row stride as the regular buffer: rows start on 16-byte boundaries
    grad = torch.full((st.R, st.grad.stride(0)), float("nan"), device="cuda")[:, :V]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    S.specopd_tv_overlap_e2e_static(st.draft, st.teacher, V, st.num_branches, W, 0.0, alpha, loss, grad, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref_alpha, ref_loss, ref_grad = ref
    a = alpha[:st.R].double().cpu().numpy()
    g = grad.double().cpu().numpy()
    assert np.max(np.abs(a - ref_alpha)) <= 1e-4
    assert abs(float(loss.item()) - ref_loss) <= 1e-4
    assert np.linalg.norm(g - ref_grad) <= 1e-3 * np.linalg.norm(ref_grad)


@pytest.mark.gpu
@pytest.mark.parametrize("dtype,B,W,V", [("bf16", 4, 16, 151936), ("f32", 3, 5, 4099)])
def test_static_scratch_matches_workspace_entry_point(dtype, B, W, V):
    """Two calls in a row against the regular entry point's results, with a
    call of another shape and seed between them, so that scratch the second
    call failed to rewrite or clear would not hold its own correct values."""
    S = _lib()
    st, ref = _case(dtype, B, W, V, seed=21)
    assert S.specopd_overlap_workspace_bytes(st.R, V, st.num_branches) <= S.STATIC_SCRATCH_BYTES
    st2, ref2 = _case(dtype, B + 2, max(1, W - 2), V - 96, seed=22)
    _static_call(S, st, V, W, ref)
    _static_call(S, st2, V - 96, max(1, W - 2), ref2)
    _static_call(S, st, V, W, ref)
