"""The seeded input recipes: determinism and the distributions the workloads describe."""
import numpy as np
import torch

import workloads as wl


def test_deterministic_and_independent_of_order():
    a1 = wl.normal((4, 5), 7, "x")
    _ = wl.normal((3,), 7, "y")
    a2 = wl.normal((4, 5), 7, "x")
    assert torch.equal(a1, a2)
    assert not torch.equal(wl.normal((4, 5), 7, "z"), a1)


def test_unit_sphere_queries():
    q = wl.unit_sphere_bf16((3, 2, 64, 128), 1, "q").double()
    n = q.pow(2).sum(-1).sqrt()
    assert torch.allclose(n, torch.ones_like(n), atol=4e-3)  # bf16 rounding of each element


def test_alpha_recipe():
    a = wl.alpha_decay((200_000,), 2, "alpha")
    assert a.dtype == torch.float32
    assert float(a.min()) >= wl.ALPHA_LO and float(a.max()) <= wl.ALPHA_HI < 1.0
    frac = float((a == np.float32(0.9)).double().mean())
    # P(sigmoid(-x) <= 0.9) for x ~ N(0,1) is P(x >= -ln 9) = Phi(2.197) ~ 0.986
    assert abs(frac - 0.986) < 0.003
    u = wl.alpha_decay((100_000,), 2, "alpha_u", mode="uniform")
    assert float((u == np.float32(0.9)).double().mean()) < 0.001


def test_beta_and_lengths():
    b = wl.beta_strength((10_000,), 3, "beta")
    assert 0.0 < float(b.min()) and float(b.max()) < 1.0
    lens = wl.mla_seq_lens(wl.CONFIGS["mla_decode_b16"])
    assert lens.dtype == torch.int32 and lens.shape == (16,)
    assert int(lens.min()) >= 8192 and int(lens.max()) <= 131072


def test_large_draws_are_sliced_consistently():
    x = wl.normal_bf16((5, 3, 4), 9, "c")
    y = wl.normal_bf16((5, 3, 4), 9, "c")
    assert torch.equal(x, y) and x.dtype == torch.bfloat16


def test_paginate_moves_rows_only():
    c = wl.normal_bf16((3, 70, 8), 1, "c")
    lens = torch.tensor([70, 0, 33], dtype=torch.int32)
    pool, bt = wl.paginate(c, lens, 32, 5, spare_pages=2)
    assert pool.shape == (3 + 2 + 2, 32, 8) and bt.shape == (3, 3)
    used = bt[bt >= 0]
    assert len(set(used.tolist())) == used.numel()   # no page used twice
    for b in range(3):
        for t in range(int(lens[b])):
            assert torch.equal(pool[bt[b, t // 32], t % 32], c[b, t])
    assert torch.isnan(pool[bt[2, 1], 1:].float()).all()   # past the length
