"""Pins for the oracle's causal convolution along tree ancestry (CPU only).

What fixes the answers:
  * on the trunk, and on each branch's own sequence (trunk through the anchor,
    then the branch's samples), the convolution is the textbook causal FIR
    filter with zero initial state, computed here by scipy.signal.lfilter;
  * an impulse on trunk token t reaches exactly the rows whose history holds t
    within Kw - 1 steps back, with the weight of that lag;
  * a branch's rows never read a sibling's tokens (siblings at one anchor);
  * the activation is torch's SiLU.
"""
import numpy as np
import pytest
import torch
from scipy.signal import lfilter

from oracle import conv as CV
from oracle import tree as T


def _case(seed=0, C=5, Kw=4):
    pt = T.pack([20, 9], [3, 2], [3, 2], [5, 5, 19, 2, 8], 4, True)
    rng = np.random.default_rng(seed)
    x = rng.normal(size=(pt.num_rows, C))
    w = rng.normal(size=(C, Kw))
    b = rng.normal(size=C)
    return pt, x, w, b


def _fir(seq, w, b):
    """Causal FIR per channel: y[t] = b + sum_j w[j] seq[t - j] (zero before the start)."""
    return np.stack([lfilter(w[c], [1.0], seq[:, c]) + b[c] for c in range(seq.shape[1])], axis=1)


def test_each_history_is_a_causal_fir():
    pt, x, w, b = _case()
    out = CV.tree_causal_conv(pt, x, w, b)
    for r in range(pt.num_rows):
        hist = CV.history(pt, r)
        np.testing.assert_allclose(out[r], _fir(x[hist], w, b)[-1], rtol=0, atol=1e-12)
    # the trunk of tree 0 as one sequence
    np.testing.assert_allclose(out[:20], _fir(x[:20], w, b), rtol=0, atol=1e-12)
    # the branch at anchor 19 continues the trunk: its rows are the FIR of x_0..x_19, y_1..y_4
    rows = [20 + 2 * 4 + i for i in range(4)]
    seq = np.concatenate([x[:20], x[rows]])
    np.testing.assert_allclose(out[rows], _fir(seq, w, b)[-4:], rtol=0, atol=1e-12)


def test_impulse_reaches_the_right_descendants():
    pt, _, w, _ = _case(C=1, Kw=4)
    t = 4
    x = np.zeros((pt.num_rows, 1))
    x[t] = 1.0
    out = CV.tree_causal_conv(pt, x, w)
    want = np.zeros(pt.num_rows)
    want[t:t + 4] = w[0, :4]                            # trunk rows t .. t+3
    for b, a in enumerate([5, 5, 19]):                   # branches of tree 0, rows 20 + 4 b + i - 1
        for i in range(1, 5):
            lag = (a - t) + i
            if 0 <= a - t and lag < 4:
                want[20 + 4 * b + i - 1] = w[0, lag]
    np.testing.assert_allclose(out[:, 0], want, rtol=0, atol=1e-15)


def test_siblings_are_isolated():
    pt, x, w, b = _case()
    base = CV.tree_causal_conv(pt, x, w, b)
    y = x.copy()
    y[20:24] += 100.0                                    # the first branch at anchor 5
    out = CV.tree_causal_conv(pt, y, w, b)
    changed = np.nonzero(np.any(np.abs(out - base) > 0, axis=1))[0]
    assert list(changed) == [20, 21, 22, 23]             # its sibling (rows 24..27) is untouched


def test_silu_is_torchs():
    pt, x, w, b = _case()
    lin = CV.tree_causal_conv(pt, x, w, b)
    act = CV.tree_causal_conv(pt, x, w, b, silu=True)
    np.testing.assert_allclose(act, torch.nn.functional.silu(torch.from_numpy(lin)).numpy(), rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("Kw", [1, 2, 8])
def test_width_one_scales_and_wide_windows_reach_the_trunk(Kw):
    pt, x, w, b = _case(Kw=Kw)
    out = CV.tree_causal_conv(pt, x, w)
    if Kw == 1:
        np.testing.assert_allclose(out, x * w[:, 0], rtol=0, atol=1e-15)
    else:
        r = 20 + 1                                       # y_{0,2} of the branch at anchor 5: x_0..x_5, y_1, y_2
        hist = [0, 1, 2, 3, 4, 5, 20, 21]
        assert CV.history(pt, r) == hist
        want = sum(w[:, j] * x[hist[-1 - j]] for j in range(min(Kw, len(hist))))
        np.testing.assert_allclose(out[r], want, rtol=0, atol=1e-12)
