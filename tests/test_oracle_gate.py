"""Pins the KDA output-gate oracle (gated RMSNorm) to torch's rms_norm and to its limits:
the gate at +inf passes torch.nn.functional.rms_norm's result; the gate at 0 halves it; the
output RMS is 1 when w = 1 and the gate is wide open; scaling the input does not change it
(eps = 0); a large negative gate closes it."""
import numpy as np
import torch

import oracle


def test_matches_torch_rms_norm_and_gate_limits():
    rng = np.random.default_rng(0)
    o = rng.standard_normal((6, 128)) * 0.3
    w = rng.uniform(0.5, 1.5, 128)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(o), (128,), torch.from_numpy(w), eps=1e-5).numpy()
    np.testing.assert_allclose(oracle.gated_rmsnorm(o, np.full_like(o, 60.0), w), ref, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(oracle.gated_rmsnorm(o, np.zeros_like(o), w), 0.5 * ref, rtol=1e-12, atol=1e-14)
    assert np.abs(oracle.gated_rmsnorm(o, np.full_like(o, -800.0), w)).max() == 0.0


def test_unit_rms_and_scale_invariance():
    rng = np.random.default_rng(1)
    o = rng.standard_normal((4, 128))
    g = rng.standard_normal((4, 128))
    y = oracle.gated_rmsnorm(o, np.full_like(o, 60.0), None, eps=0.0)
    np.testing.assert_allclose(np.sqrt(np.mean(y ** 2, axis=1)), 1.0, rtol=1e-12)
    np.testing.assert_allclose(oracle.gated_rmsnorm(7.5 * o, g, None, eps=0.0), oracle.gated_rmsnorm(o, g, None, eps=0.0),
                               rtol=1e-12)
