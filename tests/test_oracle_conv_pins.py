"""Pins of the oracle's short convolution (depthwise, causal, width K, then SiLU) against what
holds independently of it: torch's grouped conv1d and SiLU, the impulse response, causality,
the sequence boundaries and the carried state."""
import numpy as np
import torch

import oracle


def _inputs(T, C, K, seed):
    rng = np.random.default_rng(seed)
    return rng.standard_normal((T, C)), rng.standard_normal((C, K))


def test_conv_matches_torch_grouped_conv1d():
    """One sequence, zero history: conv1d with groups = C on the input left-padded by K - 1
    zeros (torch computes a cross-correlation, i.e. weight[c, j] meets x[t - (K - 1) + j])."""
    for K in (1, 2, 3, 4):
        x, w = _inputs(37, 5, K, seed=K)
        y, _ = oracle.short_conv1d_silu(x, w)
        xt = torch.from_numpy(x.T[None]).double()                       # [1, C, T]
        pre = torch.nn.functional.conv1d(torch.nn.functional.pad(xt, (K - 1, 0)),
                                         torch.from_numpy(w[:, None, :]).double(), groups=w.shape[0])
        ref = torch.nn.functional.silu(pre)[0].T.numpy()
        np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_conv_impulse_response():
    T, C, K, t0 = 12, 3, 4, 5
    _, w = _inputs(T, C, K, seed=9)
    x = np.zeros((T, C))
    x[t0] = 1.0
    y, _ = oracle.short_conv1d_silu(x, w)
    for t in range(T):
        m = t - t0
        pre = w[:, K - 1 - m] if 0 <= m < K else np.zeros(C)
        np.testing.assert_allclose(y[t], torch.nn.functional.silu(torch.from_numpy(pre)).numpy(), rtol=1e-14, atol=0)


def test_conv_is_causal():
    x, w = _inputs(20, 4, 4, seed=3)
    y, _ = oracle.short_conv1d_silu(x, w)
    x2 = x.copy()
    x2[11] += 5.0
    y2, _ = oracle.short_conv1d_silu(x2, w)
    np.testing.assert_array_equal(y2[:11], y[:11])
    assert np.abs(y2[11:15] - y[11:15]).max() > 1e-3
    np.testing.assert_array_equal(y2[15:], y[15:])


def test_conv_varlen_is_separate_runs():
    x, w = _inputs(30, 3, 4, seed=5)
    cu = np.array([0, 2, 9, 9, 30])
    y, f = oracle.short_conv1d_silu(x, w, cu_seqlens=cu)
    for n in range(4):
        a, b = cu[n], cu[n + 1]
        yn, fn = oracle.short_conv1d_silu(x[a:b], w)
        np.testing.assert_array_equal(y[a:b], yn)
        np.testing.assert_array_equal(f[n], fn[0])


def test_conv_state_composition():
    """A prefix run's final state carried into the rest equals one run over everything, token
    by token (the decode recurrence) included; a sequence shorter than K - 1 keeps part of the
    carried history."""
    x, w = _inputs(25, 4, 4, seed=7)
    y, f = oracle.short_conv1d_silu(x, w)
    for cut in (1, 2, 3, 10, 24):
        y1, f1 = oracle.short_conv1d_silu(x[:cut], w)
        y2, f2 = oracle.short_conv1d_silu(x[cut:], w, initial_state=f1)
        np.testing.assert_allclose(np.concatenate([y1, y2]), y, rtol=1e-14, atol=1e-15)
        np.testing.assert_array_equal(f2, f)
    state = np.zeros((1, 3, 4))
    for t in range(25):
        yt, state = oracle.short_conv1d_silu(x[t:t + 1], w, initial_state=state)
        np.testing.assert_allclose(yt[0], y[t], rtol=1e-14, atol=1e-15)


def test_conv_width_one_is_pointwise():
    x, w = _inputs(9, 6, 1, seed=2)
    y, f = oracle.short_conv1d_silu(x, w)
    pre = x * w[:, 0]
    np.testing.assert_allclose(y, pre / (1.0 + np.exp(-pre)), rtol=1e-15)
    assert f.shape == (1, 0, 6)
