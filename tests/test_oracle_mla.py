"""Pins the gated latent-attention oracle.

- absorbed (576-wide query against the latent rows) equals expanded attention, run by torch's
  scaled_dot_product_attention in fp64 on explicit per-head keys [W_UK^T c ; rope] and values
  W_UV^T c, with random W_UK / W_UV;
- a brute-force softmax (scipy) on tiny inputs, and log-sum-exp against scipy;
- special cases: one cached row, identical rows, zero length, rows past the length ignored,
  the sigmoid gate.
"""
import numpy as np
import pytest
import torch
from scipy.special import expit, logsumexp, softmax

import oracle


def _bf16_round(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)


def _bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _cache(rng, B, L, D):
    c = _bf16_round(rng.standard_normal((B, L, D)))
    return c.to(torch.float64).numpy(), _bits(c)


def test_absorbed_equals_expanded_attention():
    rng = np.random.default_rng(0)
    B, H, Dc, Dr, dn, dvh, L = 2, 3, 32, 8, 12, 10, 17
    scale = 1.0 / np.sqrt(dn + Dr)
    c, bits = _cache(rng, B, L, Dc + Dr)
    W_UK = rng.standard_normal((H, Dc, dn)) / np.sqrt(Dc)
    W_UV = rng.standard_normal((H, Dc, dvh)) / np.sqrt(Dc)
    q_nope = rng.standard_normal((B, H, dn))
    q_rope = rng.standard_normal((B, H, Dr))
    lens = np.array([L, 9], dtype=np.int32)
    gate = rng.standard_normal((B, H))

    # absorbed: q_abs = [W_UK q_nope ; q_rope], attention over raw latent rows, then W_UV^T
    q_abs = np.concatenate([np.einsum("hcn,bhn->bhc", W_UK, q_nope), q_rope], axis=-1)
    o_lat, _ = oracle.mla_decode(q_abs, bits, lens, gate, scale=scale, d_latent=Dc)
    o_abs = np.einsum("hcv,bhc->bhv", W_UV, o_lat)

    # expanded: per-head keys and values, plain softmax attention by torch
    for b in range(B):
        Lb = int(lens[b])
        cl = torch.from_numpy(c[b, :Lb])
        K = torch.cat([torch.einsum("hcn,tc->htn", torch.from_numpy(W_UK), cl[:, :Dc]),
                       cl[None, :, Dc:].expand(H, Lb, Dr)], dim=-1)
        V = torch.einsum("hcv,tc->htv", torch.from_numpy(W_UV), cl[:, :Dc])
        Q = torch.cat([torch.from_numpy(q_nope[b]), torch.from_numpy(q_rope[b])], dim=-1)[:, None, :]
        ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V, scale=scale)[:, 0, :].numpy()
        ref = ref * expit(gate[b])[:, None]
        np.testing.assert_allclose(o_abs[b], ref, rtol=0, atol=1e-12)


def test_brute_force_softmax_and_lse():
    rng = np.random.default_rng(1)
    B, H, Dc, Dr, L = 3, 4, 16, 4, 13
    c, bits = _cache(rng, B, L, Dc + Dr)
    q = rng.standard_normal((B, H, Dc + Dr))
    lens = np.array([13, 1, 6], dtype=np.int32)
    scale = 0.37
    o, lse = oracle.mla_decode(q, bits, lens, None, scale=scale, d_latent=Dc)
    for b in range(B):
        Lb = lens[b]
        s = scale * q[b] @ c[b, :Lb].T          # [H, Lb]
        p = softmax(s, axis=-1)
        np.testing.assert_allclose(o[b], p @ c[b, :Lb, :Dc], rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse[b], logsumexp(s, axis=-1), rtol=0, atol=1e-13)


def test_one_row_and_identical_rows():
    rng = np.random.default_rng(2)
    H, Dc, Dr = 5, 16, 8
    c, bits = _cache(rng, 1, 1, Dc + Dr)
    q = rng.standard_normal((1, H, Dc + Dr))
    g = rng.standard_normal((1, H))
    o, _ = oracle.mla_decode(q, bits, np.array([1], np.int32), g, scale=1.0, d_latent=Dc)
    np.testing.assert_allclose(o[0], expit(g[0])[:, None] * c[0, 0, :Dc][None, :], rtol=1e-15, atol=0)
    rep = np.repeat(bits, 40, axis=1)
    o2, lse2 = oracle.mla_decode(q, rep, np.array([40], np.int32), g, scale=1.0, d_latent=Dc)
    np.testing.assert_allclose(o2, o, rtol=1e-13, atol=1e-15)
    s0 = q[0] @ c[0, 0]
    np.testing.assert_allclose(lse2[0], s0 + np.log(40.0), rtol=1e-13)


def test_zero_length_and_rows_past_length():
    rng = np.random.default_rng(3)
    H, Dc, Dr, L = 2, 8, 4, 10
    c, bits = _cache(rng, 2, L, Dc + Dr)
    q = rng.standard_normal((2, H, Dc + Dr))
    lens = np.array([0, 6], np.int32)
    o, lse = oracle.mla_decode(q, bits, lens, None, scale=0.5, d_latent=Dc)
    assert np.array_equal(o[0], np.zeros((H, Dc))) and np.all(np.isneginf(lse[0]))
    junk = bits.copy()
    junk[1, 6:] = _bits(_bf16_round(np.full((L - 6, Dc + Dr), 1e30)))
    o2, lse2 = oracle.mla_decode(q, junk, lens, None, scale=0.5, d_latent=Dc)
    assert np.array_equal(o2, o) and np.array_equal(lse2[1], lse[1])


def test_gate_limits():
    rng = np.random.default_rng(4)
    H, Dc, Dr, L = 3, 8, 4, 7
    c, bits = _cache(rng, 1, L, Dc + Dr)
    q = rng.standard_normal((1, H, Dc + Dr))
    lens = np.array([L], np.int32)
    o_none, _ = oracle.mla_decode(q, bits, lens, None, scale=0.3, d_latent=Dc)
    o_zero, _ = oracle.mla_decode(q, bits, lens, np.zeros((1, H)), scale=0.3, d_latent=Dc)
    o_big, _ = oracle.mla_decode(q, bits, lens, np.full((1, H), 60.0), scale=0.3, d_latent=Dc)
    np.testing.assert_allclose(o_zero, 0.5 * o_none, rtol=1e-15)
    np.testing.assert_allclose(o_big, o_none, rtol=1e-15)


@pytest.mark.parametrize("nthreads", [1, 3])
def test_threads_do_not_change_results(nthreads):
    rng = np.random.default_rng(5)
    c, bits = _cache(rng, 3, 20, 24)
    q = rng.standard_normal((3, 4, 24))
    lens = np.array([20, 3, 11], np.int32)
    o1, l1 = oracle.mla_decode(q, bits, lens, None, scale=0.2, d_latent=16, nthreads=1)
    on, ln = oracle.mla_decode(q, bits, lens, None, scale=0.2, d_latent=16, nthreads=nthreads)
    assert np.array_equal(o1, on) and np.array_equal(l1, ln)


def _paginate(rng, bits, lens, P, extra_pages=3):
    """Scatters each sequence's rows into pages of P rows at random pool positions; the pool's
    unused rows hold NaN bit patterns. Returns (pool bits, block table)."""
    B, L, D = bits.shape
    per_seq = [(int(n) + P - 1) // P for n in lens]
    n_pages = sum(per_seq) + extra_pages
    perm = rng.permutation(n_pages)
    pool = np.full((n_pages, P, D), 0x7FC0, np.uint16)
    bt = np.full((B, max(max(per_seq), 1) + 1), -1, np.int32)
    k = 0
    for b in range(B):
        for j in range(per_seq[b]):
            pg = int(perm[k])
            k += 1
            bt[b, j] = pg
            rows = bits[b, j * P:min((j + 1) * P, int(lens[b]))]
            pool[pg, :rows.shape[0]] = rows
    return pool, bt


def test_paged_equals_contiguous_and_brute_force():
    """The paged layout only moves rows: with pages scattered through a pool (unused rows NaN),
    the result equals the contiguous cache's bit for bit, and a scipy softmax over the rows
    gathered through the block table."""
    rng = np.random.default_rng(6)
    H, Dc, Dr, L, P = 3, 16, 8, 23, 4
    c, bits = _cache(rng, 3, L, Dc + Dr)
    q = rng.standard_normal((3, H, Dc + Dr))
    gate = rng.standard_normal((3, H))
    lens = np.array([23, 0, 9], np.int32)
    pool, bt = _paginate(rng, bits, lens, P)
    o_c, l_c = oracle.mla_decode(q, bits, lens, gate, scale=0.4, d_latent=Dc)
    o_p, l_p = oracle.mla_decode_paged(q, pool, bt, lens, gate, scale=0.4, d_latent=Dc)
    assert np.array_equal(o_p, o_c) and np.array_equal(l_p, l_c)
    pool_f = torch.from_numpy(pool.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    for b in (0, 2):
        rows = np.stack([pool_f[bt[b, t // P], t % P] for t in range(lens[b])])
        s = 0.4 * q[b] @ rows.T
        ref = softmax(s, axis=1) @ rows[:, :Dc] * expit(gate[b])[:, None]
        np.testing.assert_allclose(o_p[b], ref, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(l_p[b], logsumexp(s, axis=1), rtol=1e-13)


def test_paged_rejects_bad_block_table():
    rng = np.random.default_rng(7)
    c, bits = _cache(rng, 1, 8, 12)
    q = rng.standard_normal((1, 2, 12))
    lens = np.array([8], np.int32)
    pool, bt = _paginate(rng, bits, lens, 4, extra_pages=0)
    bad = bt.copy()
    bad[0, 1] = pool.shape[0]
    with pytest.raises(RuntimeError):
        oracle.mla_decode_paged(q, pool, bad, lens, None, scale=0.5, d_latent=8)
    with pytest.raises(RuntimeError):
        oracle.mla_decode_paged(q, pool, bt[:, :1], lens, None, scale=0.5, d_latent=8)
