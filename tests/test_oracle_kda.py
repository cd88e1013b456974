"""Pins the KDA oracle (token-by-token and chunked) to facts fixed outside itself.

- the product form S_t = (I - beta k k^T) Diag(alpha) S_{t-1} + beta k v^T, expanded with explicit
  matrices on tiny shapes (d_k != d_v so that a transposed operand fails);
- special cases: alpha = 1, beta = 0 keeps the state; unit k with beta = 1 makes S_t^T k_t = v_t;
  beta = 0 is pure decay with a closed form; one token from zero state gives beta k v^T;
- the chunked (WY/UT) form agrees with the token-by-token form;
- L2 normalisation against numpy's norm.
"""
import numpy as np
import pytest

import oracle


def _rand_inputs(rng, B, T, H, dk, dv, alpha_lo=0.5, unit_k=False, s0_std=0.3):
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    if unit_k:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    alpha = rng.uniform(alpha_lo, 1.0, (B, T, H, dk))
    beta = rng.uniform(0.05, 1.0, (B, T, H))
    S0 = s0_std * rng.standard_normal((B, H, dk, dv))
    return q, k, v, alpha, beta, S0


def _brute_force(q, k, v, alpha, beta, S0, scale):
    """Explicit-matrix product form of the gated delta rule, one (b, h) at a time."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    S = S0.copy()
    for b in range(B):
        for h in range(H):
            M = S[b, h]
            for t in range(T):
                kt = k[b, t, h][:, None]
                P = np.eye(dk) - beta[b, t, h] * (kt @ kt.T)
                M = P @ np.diag(alpha[b, t, h]) @ M + beta[b, t, h] * (kt @ v[b, t, h][None, :])
                o[b, t, h] = scale * (M.T @ q[b, t, h])
            S[b, h] = M
    return o, S


@pytest.mark.parametrize("dk,dv,T", [(4, 4, 6), (3, 5, 5), (5, 2, 4), (1, 3, 3)])
def test_recurrent_matches_product_form(dk, dv, T):
    rng = np.random.default_rng(10 + dk * 7 + dv)
    q, k, v, a, b, S0 = _rand_inputs(rng, 2, T, 3, dk, dv)
    o, S = oracle.kda_recurrent(q, k, v, a, b, S0, scale=0.7)
    o_ref, S_ref = _brute_force(q, k, v, a, b, S0, 0.7)
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(S, S_ref, rtol=0, atol=1e-12)


def test_pin_rejects_plausible_mistakes():
    """The product-form pin separates the oracle from nearby wrong recurrences."""
    rng = np.random.default_rng(3)
    dk, dv, T = 3, 5, 5
    q, k, v, a, b, S0 = _rand_inputs(rng, 1, T, 1, dk, dv)
    o, S = oracle.kda_recurrent(q, k, v, a, b, S0)

    def wrong(variant):
        M = S0[0, 0].copy()
        for t in range(T):
            kt, vt, at, bt = k[0, t, 0], v[0, t, 0], a[0, t, 0], b[0, t, 0]
            Md = np.diag(at) @ M
            if variant == "delta_before_decay":
                M = np.diag(at) @ (M + np.outer(kt, bt * (vt - M.T @ kt)))
            elif variant == "predict_from_undecayed":
                M = Md + np.outer(kt, bt * (vt - M.T @ kt))
            elif variant == "sign":
                M = Md + np.outer(kt, bt * (vt + Md.T @ kt))
            elif variant == "no_strength_on_prediction":
                M = Md + np.outer(kt, bt * vt - Md.T @ kt)
        return M

    for variant in ("delta_before_decay", "predict_from_undecayed", "sign", "no_strength_on_prediction"):
        assert np.abs(wrong(variant) - S[0, 0]).max() > 1e-3, variant


def test_identity_step_keeps_state_exactly():
    rng = np.random.default_rng(1)
    q, k, v, a, b, S0 = _rand_inputs(rng, 2, 4, 3, 8, 6)
    a[:] = 1.0
    b[:] = 0.0
    o, S = oracle.kda_recurrent(q, k, v, a, b, S0, scale=1.0)
    assert np.array_equal(S, S0)
    for t in range(4):
        np.testing.assert_allclose(o[:, t], np.einsum("bhij,bhi->bhj", S0, q[:, t]), rtol=0, atol=1e-13)


def test_unit_key_full_strength_write_is_exact():
    """With ||k|| = 1 and beta = 1 the written state maps k_t to v_t, whatever alpha and S."""
    rng = np.random.default_rng(2)
    q, k, v, a, b, S0 = _rand_inputs(rng, 1, 1, 4, 16, 16, unit_k=True)
    b[:] = 1.0
    for T in (1,):
        o, S = oracle.kda_recurrent(q, k, v, a, b, S0)
        for h in range(4):
            np.testing.assert_allclose(S[0, h].T @ k[0, 0, h], v[0, 0, h], rtol=0, atol=1e-12)


def test_zero_strength_is_pure_decay():
    rng = np.random.default_rng(4)
    q, k, v, a, b, S0 = _rand_inputs(rng, 1, 7, 2, 6, 4)
    b[:] = 0.0
    o, S = oracle.kda_recurrent(q, k, v, a, b, S0)
    gtot = np.prod(a, axis=1)  # [B,H,dk]
    np.testing.assert_allclose(S, gtot[..., None] * S0, rtol=1e-14, atol=0)


def test_one_token_from_zero_state():
    rng = np.random.default_rng(5)
    q, k, v, a, b, _ = _rand_inputs(rng, 1, 1, 3, 5, 7)
    S0 = np.zeros((1, 3, 5, 7))
    o, S = oracle.kda_recurrent(q, k, v, a, b, S0, scale=0.25)
    for h in range(3):
        kk, vv, qq, bb = k[0, 0, h], v[0, 0, h], q[0, 0, h], b[0, 0, h]
        np.testing.assert_allclose(S[0, h], bb * np.outer(kk, vv), rtol=0, atol=1e-14)
        np.testing.assert_allclose(o[0, 0, h], 0.25 * bb * (kk @ qq) * vv, rtol=0, atol=1e-14)


@pytest.mark.parametrize("T,C,dk,dv", [(32, 8, 16, 16), (37, 8, 6, 10), (5, 8, 4, 4), (24, 1, 3, 3),
                                       (64, 16, 8, 12), (19, 64, 5, 5)])
def test_chunked_equals_recurrent(T, C, dk, dv):
    rng = np.random.default_rng(T * 100 + C)
    q, k, v, a, b, S0 = _rand_inputs(rng, 2, T, 2, dk, dv, alpha_lo=0.7)
    o1, S1 = oracle.kda_recurrent(q, k, v, a, b, S0, scale=0.5)
    o2, S2 = oracle.kda_chunked(q, k, v, a, b, S0, chunk=C, scale=0.5)
    np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-11 * max(1.0, np.abs(o1).max()))
    np.testing.assert_allclose(S2, S1, rtol=0, atol=1e-11 * max(1.0, np.abs(S1).max()))


def test_chunked_equals_recurrent_full_head_dim():
    """The shape of the workloads: d = 128, chunk 64, decays in [0.9, 1), T with a ragged tail."""
    rng = np.random.default_rng(77)
    q, k, v, a, b, S0 = _rand_inputs(rng, 1, 150, 2, 128, 128, alpha_lo=0.9, unit_k=True, s0_std=0.02)
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    o1, S1 = oracle.kda_recurrent(q, k, v, a, b, S0)
    o2, S2 = oracle.kda_chunked(q, k, v, a, b, S0, chunk=64)
    np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-10)
    np.testing.assert_allclose(S2, S1, rtol=0, atol=1e-10)


def test_multi_thread_is_identical():
    rng = np.random.default_rng(6)
    q, k, v, a, b, S0 = _rand_inputs(rng, 3, 9, 5, 8, 8)
    o1, S1 = oracle.kda_recurrent(q, k, v, a, b, S0, nthreads=1)
    o4, S4 = oracle.kda_recurrent(q, k, v, a, b, S0, nthreads=4)
    assert np.array_equal(o1, o4) and np.array_equal(S1, S4)


def test_l2norm_against_numpy_norm():
    rng = np.random.default_rng(8)
    x = rng.standard_normal((7, 3, 128))
    y = oracle.l2norm(x, eps=0.0)
    np.testing.assert_allclose(y, x / np.linalg.norm(x, axis=-1, keepdims=True), rtol=1e-14, atol=0)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), 1.0, rtol=1e-14)
    # eps only matters for tiny vectors
    z = np.zeros((1, 128))
    z[0, 0] = 1e-4
    assert abs(oracle.l2norm(z, eps=1e-6)[0, 0] - 1e-4 / np.sqrt(1e-8 + 1e-6)) < 1e-15
