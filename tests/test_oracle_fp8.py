"""Pins the FP8 (E4M3) parts of the oracle: the code <-> value maps, the attention over an FP8
cache and the FP8 cache rows.

- decode: every one of the 256 codes against torch's float8_e4m3fn (an independent library
  implementation of the format), plus the format's fixed points (largest finite 448, smallest
  normal 2^-6, smallest subnormal 2^-9, the NaN patterns, signed zero);
- encode: against torch on fp32 values inside the finite range; brute force "nearest code, ties to
  the even code" over every finite code for random and midpoint inputs; saturation and NaN;
  round trip of every finite code;
- attention over an FP8 cache equals the (separately pinned) bf16-cache attention when the scale
  is a power of two (every dequantised element is then exactly a bf16 value), and equals a
  torch fp64 softmax for a general scale; the paged form equals the contiguous one;
- FP8 cache rows: the fp32 quotient rounded by torch, latent and RoPE parts.
"""
import numpy as np
import pytest
import torch

import oracle
from workloads import paginate


def _torch_decode(codes):
    return torch.from_numpy(np.asarray(codes, dtype=np.uint8)).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def _torch_encode_f32(x32):
    """torch's float32 -> E4M3 conversion (round to nearest even; no saturation, so only inputs
    inside the finite range are compared)."""
    return torch.from_numpy(np.asarray(x32, dtype=np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


ALL = np.arange(256, dtype=np.uint8)
FINITE = ALL[(ALL & 0x7F) != 0x7F]


def test_decode_matches_library_on_every_code():
    mine = oracle.e4m3_decode(ALL)
    ref = _torch_decode(ALL)
    nan = (ALL & 0x7F) == 0x7F
    assert np.isnan(mine[nan]).all() and np.isnan(ref[nan]).all()
    np.testing.assert_array_equal(mine[~nan], ref[~nan])
    assert np.array_equal(np.signbit(mine[~nan]), np.signbit(ref[~nan]))


def test_decode_fixed_points():
    v = oracle.e4m3_decode(np.array([0x7E, 0xFE, 0x08, 0x07, 0x01, 0x38, 0x00, 0x80], dtype=np.uint8))
    assert v[0] == 448.0 and v[1] == -448.0
    assert v[2] == 2.0 ** -6 and v[3] == 7 * 2.0 ** -9 and v[4] == 2.0 ** -9 and v[5] == 1.0
    assert v[6] == 0.0 and not np.signbit(v[6]) and v[7] == 0.0 and np.signbit(v[7])
    pos = oracle.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8))
    assert (np.diff(pos) > 0).all()  # codes 0..126 increase strictly


def test_encode_round_trips_every_finite_code():
    vals = oracle.e4m3_decode(FINITE)
    np.testing.assert_array_equal(oracle.e4m3_encode(vals), FINITE)


def test_encode_matches_library_in_range():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.standard_normal(20000) * s for s in (1e-3, 0.05, 1.0, 20.0, 150.0)])
    x = x.astype(np.float32)
    x = x[np.abs(x) < 448]
    # midpoints between neighbouring codes (exact in fp32), both signs
    pos = oracle.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8))
    mids = ((pos[1:] + pos[:-1]) / 2).astype(np.float32)
    x = np.concatenate([x, mids, -mids])
    np.testing.assert_array_equal(oracle.e4m3_encode(x.astype(np.float64)), _torch_encode_f32(x))


def test_encode_is_nearest_with_ties_to_even_brute_force():
    rng = np.random.default_rng(2)
    grid = oracle.e4m3_decode(FINITE)
    pos = oracle.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8))
    x = np.concatenate([rng.uniform(-448, 448, 3000), rng.uniform(-0.05, 0.05, 3000),
                        (pos[1:] + pos[:-1]) / 2, -(pos[1:] + pos[:-1]) / 2])
    codes = oracle.e4m3_encode(x)
    got = oracle.e4m3_decode(codes)
    for xi, ci, gi in zip(x, codes, got):
        d = np.abs(grid - xi)
        best = d.min()
        assert abs(gi - xi) == best
        if np.count_nonzero(d == best) > 1 and gi != 0.0:  # a tie: the even code (mantissa LSB 0)
            assert (int(ci) & 1) == 0


def test_encode_saturates_and_keeps_nan():
    c = oracle.e4m3_encode(np.array([448.0, 449.0, 464.0, 500.0, 1e30, -1e30, np.inf, -np.inf, np.nan,
                                     2.0 ** -10, 3 * 2.0 ** -10, -0.0, -(2.0 ** -11)]))
    assert list(c[:8]) == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0x7E, 0xFE]
    assert c[8] == 0x7F
    assert c[9] == 0x00  # halfway between 0 and 2^-9: the even code, 0
    assert c[10] == 0x02  # halfway between 2^-9 and 2^-8: code 2 (even)
    assert c[11] == 0x80 and c[12] == 0x80  # signed zeros


def _fp8_cache(rng, B, L, D, spread=2.0):
    x = rng.standard_normal((B, L, D)) * spread
    return oracle.e4m3_encode(x)


def test_fp8_attention_equals_bf16_attention_for_power_of_two_scale():
    rng = np.random.default_rng(3)
    B, H, Dc, Dr, L = 2, 4, 32, 8, 21
    codes = _fp8_cache(rng, B, L, Dc + Dr)
    kv_scale = 2.0 ** -3
    vals = oracle.e4m3_decode(codes) * kv_scale  # exact in bf16 (4 significant bits)
    bits = torch.from_numpy(vals.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy(), vals)
    q = rng.standard_normal((B, H, Dc + Dr))
    lens = np.array([L, 13], dtype=np.int32)
    gate = rng.standard_normal((B, H))
    o8, l8 = oracle.mla_decode_fp8(q, codes, kv_scale, lens, gate=gate, scale=0.3, d_latent=Dc)
    ob, lb = oracle.mla_decode(q, bits, lens, gate=gate, scale=0.3, d_latent=Dc)
    np.testing.assert_array_equal(o8, ob)
    np.testing.assert_array_equal(l8, lb)


def test_fp8_attention_matches_torch_softmax_general_scale():
    rng = np.random.default_rng(4)
    B, H, Dc, Dr, L = 3, 5, 24, 8, 17
    codes = _fp8_cache(rng, B, L, Dc + Dr)
    kv_scale = 0.0371
    q = rng.standard_normal((B, H, Dc + Dr))
    lens = np.array([L, 1, 0], dtype=np.int32)
    o, lse = oracle.mla_decode_fp8(q, codes, kv_scale, lens, scale=0.25, d_latent=Dc)
    c = torch.from_numpy(_torch_decode(codes)) * kv_scale
    for b in range(B):
        n = int(lens[b])
        if n == 0:
            assert (o[b] == 0).all() and np.isneginf(lse[b]).all()
            continue
        s = 0.25 * torch.einsum("hd,td->ht", torch.from_numpy(q[b]), c[b, :n])
        p = torch.softmax(s, dim=-1)
        np.testing.assert_allclose(o[b], (p @ c[b, :n, :Dc]).numpy(), rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(lse[b], torch.logsumexp(s, dim=-1).numpy(), rtol=1e-12)


def test_fp8_paged_equals_contiguous():
    rng = np.random.default_rng(5)
    B, H, Dc, Dr, P = 3, 2, 16, 8, 4
    lens = np.array([9, 4, 13], dtype=np.int32)
    codes = _fp8_cache(rng, B, int(lens.max()), Dc + Dr)
    q = rng.standard_normal((B, H, Dc + Dr))
    pages, bt = paginate(torch.from_numpy(codes), torch.from_numpy(lens), P, seed=6, spare_pages=3)
    pages, bt = pages.numpy(), bt.numpy()
    o1, l1 = oracle.mla_decode_fp8(q, codes, 0.5, lens, scale=0.2, d_latent=Dc)
    o2, l2 = oracle.mla_decode_paged_fp8(q, pages, 0.5, bt, lens, scale=0.2, d_latent=Dc)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


@pytest.mark.parametrize("interleaved", [False, True])
def test_fp8_cache_rows_match_library_quantisation(interleaved):
    rng = np.random.default_rng(7)
    n, Dc, Dr = 6, 32, 16
    c_kv = torch.from_numpy(rng.standard_normal((n, Dc)).astype(np.float32)).to(torch.bfloat16)
    k_pe = torch.from_numpy(rng.standard_normal((n, Dr)).astype(np.float32)).to(torch.bfloat16)
    pos = rng.integers(0, 1 << 20, n)
    kv_scale = 0.0173  # |x| / kv_scale stays well inside +-448
    bits = lambda t: t.view(torch.int16).numpy().view(np.uint16)
    got = oracle.mla_cache_row_fp8(bits(c_kv), bits(k_pe), pos, kv_scale, interleaved=interleaved)
    s32 = np.float32(kv_scale)
    lat = (c_kv.float().numpy() / s32).astype(np.float32)
    turned = oracle.rope(k_pe.double().numpy(), pos, interleaved=interleaved).astype(np.float32)
    rp = (turned / s32).astype(np.float32)
    assert np.abs(lat).max() < 448 and np.abs(rp).max() < 448
    np.testing.assert_array_equal(got[:, :Dc], _torch_encode_f32(lat))
    np.testing.assert_array_equal(got[:, Dc:], _torch_encode_f32(rp))
