"""Pins the rotary-embedding oracle (the 64-wide RoPE part of latent attention) to what defines
a rotary embedding rather than to its own formula:
- a closed-form value at D = 4;
- position 0 is the identity; every pair keeps its norm;
- rotations compose: R(p) R(s) = R(p + s);
- the relative-position property <R(p) q, R(s) k> = <R(p - s) q, k>;
- the two pairings are the same rotation up to a fixed permutation of the dimensions."""
import numpy as np
import pytest

import oracle


def test_closed_form_d4():
    # pair 0 turns by p * 100^0 = 1 rad, pair 1 by p * 100^(-1/2) = 0.1 rad (p = 1)
    x = np.array([[1.0, 2.0, 3.0, 4.0]])
    y = oracle.rope(x, [1], theta=100.0)
    c0, s0, c1, s1 = np.cos(1.0), np.sin(1.0), np.cos(0.1), np.sin(0.1)
    want = [1 * c0 - 3 * s0, 2 * c1 - 4 * s1, 3 * c0 + 1 * s0, 4 * c1 + 2 * s1]
    np.testing.assert_allclose(y[0], want, rtol=0, atol=1e-15)
    yi = oracle.rope(x, [1], theta=100.0, interleaved=True)
    want_i = [1 * c0 - 2 * s0, 2 * c0 + 1 * s0, 3 * c1 - 4 * s1, 4 * c1 + 3 * s1]
    np.testing.assert_allclose(yi[0], want_i, rtol=0, atol=1e-15)


@pytest.mark.parametrize("interleaved", [False, True])
def test_identity_norms_composition(interleaved):
    rng = np.random.default_rng(0)
    x = rng.standard_normal((5, 64))
    assert np.array_equal(oracle.rope(x, [0] * 5, interleaved=interleaved), x)
    p = np.array([1, 7, 1000, 262143, 999999])
    y = oracle.rope(x, p, interleaved=interleaved)
    if interleaved:
        nx, ny = x[:, 0::2] ** 2 + x[:, 1::2] ** 2, y[:, 0::2] ** 2 + y[:, 1::2] ** 2
    else:
        nx, ny = x[:, :32] ** 2 + x[:, 32:] ** 2, y[:, :32] ** 2 + y[:, 32:] ** 2
    np.testing.assert_allclose(ny, nx, rtol=1e-12)
    s = np.array([3, 11, 17, 5, 123456])
    np.testing.assert_allclose(oracle.rope(oracle.rope(x, s, interleaved=interleaved), p, interleaved=interleaved),
                               oracle.rope(x, p + s, interleaved=interleaved), rtol=0, atol=1e-8)


@pytest.mark.parametrize("interleaved", [False, True])
def test_relative_position(interleaved):
    rng = np.random.default_rng(1)
    q, k = rng.standard_normal((6, 64)), rng.standard_normal((6, 64))
    p = np.array([10, 500, 4096, 70000, 262143, 1000000])
    s = np.array([3, 499, 100, 69999, 1, 999000])
    lhs = np.sum(oracle.rope(q, p, interleaved=interleaved) * oracle.rope(k, s, interleaved=interleaved), axis=1)
    rhs = np.sum(oracle.rope(q, p - s, interleaved=interleaved) * k, axis=1)
    np.testing.assert_allclose(lhs, rhs, rtol=0, atol=1e-8)


def test_pairings_are_a_permutation_apart():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((4, 64))
    perm = np.array([j for i in range(32) for j in (i, i + 32)])   # interleaved slot -> rotate-half slot
    p = [0, 5, 77, 300000]
    a = oracle.rope(x[:, perm], p, interleaved=True)
    b = oracle.rope(x, p)[:, perm]
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-14)


def _f32_to_bf16_bits_rne(x32):
    import torch
    return torch.from_numpy(np.asarray(x32, dtype=np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_bf16_rounding_ties_and_neighbours():
    """The oracle's rounding to bf16: exact values stay, halfway cases go to the even neighbour,
    values a hair off halfway go to the nearer one; on float32 inputs it agrees with torch."""
    one, ulp = 1.0, 2.0 ** -7
    cases = {one: 0x3F80, one + ulp / 2: 0x3F80, one + 1.5 * ulp: 0x3F82, one + ulp / 2 + 1e-12: 0x3F81,
             one + ulp / 2 - 1e-12: 0x3F80, -(one + 1.5 * ulp): 0xBF82, 0.0: 0x0000, 3.0e38: 0x7F62}
    got = oracle.round_bf16_bits(np.array(list(cases)))
    assert [int(g) for g in got] == list(cases.values())
    rng = np.random.default_rng(3)
    x32 = (rng.standard_normal(20000) * np.exp(rng.uniform(-20, 20, 20000))).astype(np.float32)
    assert np.array_equal(oracle.round_bf16_bits(x32.astype(np.float64)), _f32_to_bf16_bits_rne(x32))


def test_cache_row_is_latent_then_rotated_key():
    rng = np.random.default_rng(4)
    c = _f32_to_bf16_bits_rne(rng.standard_normal((3, 512)))
    k = _f32_to_bf16_bits_rne(rng.standard_normal((3, 64)))
    pos = [0, 17, 999999]
    rows = oracle.mla_cache_row(c, k, pos)
    assert np.array_equal(rows[:, :512], c)
    assert np.array_equal(rows[0, 512:], k[0])             # position 0: the key as given
    kf = k.astype(np.uint32) << 16
    kd = kf.view(np.float32).astype(np.float64)
    assert np.array_equal(rows[:, 512:], oracle.round_bf16_bits(oracle.rope(kd, pos)))
