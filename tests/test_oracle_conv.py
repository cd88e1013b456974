"""Pins the short-convolution oracle: impulse response, numpy.convolve, SiLU, the tail shift."""
import numpy as np
import torch

import oracle


def _run(xs, w, bias=None, silu=False):
    """Feed the tokens xs[t] ([B, Cch]) one decode step at a time from a zero tail."""
    T, B, Cch = xs.shape
    K = w.shape[1]
    tail = np.zeros((B, K - 1, Cch))
    ys = []
    for t in range(T):
        y, tail = oracle.short_conv_step(xs[t], tail, w, bias, silu)
        ys.append(y)
    return np.stack(ys), tail


def test_impulse_response_is_the_taps():
    rng = np.random.default_rng(0)
    Cch, K = 5, 4
    w = rng.standard_normal((Cch, K))
    xs = np.zeros((6, 1, Cch))
    xs[1, 0, :] = 1.0
    ys, _ = _run(xs, w)
    # one step after the impulse the newest tap applies first, then the older ones
    for lag in range(K):
        np.testing.assert_array_equal(ys[1 + lag, 0], w[:, K - 1 - lag])
    np.testing.assert_array_equal(ys[0, 0], 0.0)
    np.testing.assert_array_equal(ys[5, 0], 0.0)


def test_matches_numpy_convolve():
    rng = np.random.default_rng(1)
    T, B, Cch, K = 11, 2, 3, 4
    xs = rng.standard_normal((T, B, Cch))
    w = rng.standard_normal((Cch, K))
    bias = rng.standard_normal(Cch)
    ys, _ = _run(xs, w, bias)
    for b in range(B):
        for c in range(Cch):
            # causal convolution: y_t = sum_i w[i] x_{t-(K-1)+i}  ==  (x * reversed(w))[t]
            full = np.convolve(xs[:, b, c], w[c, ::-1])[:T] + bias[c]
            np.testing.assert_allclose(ys[:, b, c], full, rtol=0, atol=1e-13)


def test_silu_matches_torch():
    rng = np.random.default_rng(2)
    xs = rng.standard_normal((5, 2, 8)) * 3
    w = rng.standard_normal((8, 4))
    lin, _ = _run(xs, w, silu=False)
    act, _ = _run(xs, w, silu=True)
    ref = torch.nn.functional.silu(torch.from_numpy(lin)).numpy()
    np.testing.assert_allclose(act, ref, rtol=1e-14, atol=1e-15)


def test_tail_keeps_last_inputs_oldest_first():
    rng = np.random.default_rng(3)
    xs = rng.standard_normal((7, 2, 6))
    w = rng.standard_normal((6, 4))
    _, tail = _run(xs, w)
    np.testing.assert_array_equal(tail, np.transpose(xs[-3:], (1, 0, 2)))
