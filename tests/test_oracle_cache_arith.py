"""Pins the cache-arithmetic oracle to the numbers the pages print (tests/golden)."""
import json
import os

import pytest

from oracle import cache_arith as ca

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "cache_arithmetic.json")))


def _round(x, digits):
    return round(x, digits)


def test_per_token_bytes():
    assert ca.latent_row_elems() * 2 == GOLD["latent_row_bytes"]["value"]
    assert ca.per_token_bytes_hybrid() == GOLD["per_token_hybrid_bytes"]["value"]
    assert ca.per_token_bytes_all_mla() == GOLD["per_token_all_mla_bytes"]["value"]
    assert ca.per_token_bytes_hybrid(with_mtp=True) == GOLD["per_token_with_mtp_bytes"]["value"]


def test_kda_state_and_tails():
    st = ca.kda_state_bytes()
    assert _round(st / 1e6, 1) == GOLD["kda_state_mb"]["value"]
    assert _round(st / 2**20, 0) == GOLD["kda_state_mib"]["value"]
    # width-4 conv keeps K-1 = 3 bf16 inputs: 9.29 MB rounds to the page's "9 MB";
    # keeping 4 inputs (12.4 MB) or fp32 tails (18.6 MB) would not.
    assert _round(ca.conv_tail_bytes() / 1e6, 0) == GOLD["conv_tails_mb"]["value"]
    assert round(ca.conv_tail_bytes() * 4 / 3 / 1e6) != GOLD["conv_tails_mb"]["value"]


def test_cache_table():
    d = GOLD["cache_table_gb"]["digits"]
    for ctx, hyb, allm in GOLD["cache_table_gb"]["rows"]:
        assert _round(ca.cache_gb(ctx, True), d) == hyb, ctx
        assert _round(ca.cache_gb(ctx, False), d) == allm, ctx


def test_ratios_and_break_even():
    r = ca.cache_gb(1_000_000, False) / ca.cache_gb(1_000_000, True)
    assert _round(r, 1) == GOLD["reduction_at_1m"]["value"]
    be = ca.break_even_tokens()
    assert abs(be - GOLD["break_even_tokens"]["value"]) / GOLD["break_even_tokens"]["value"] < GOLD["break_even_tokens"]["rel_tol"]


def test_mha_comparison():
    b = ca.mha_bytes_per_token()
    assert _round(b / 1e6, 2) == GOLD["mha_mb_per_token"]["value"]
    assert _round(b * 1e6 / 1e12, 1) == GOLD["mha_tb_at_1m"]["value"]


def test_serving_concurrency():
    budget = ca.serving_budget_bytes()
    assert _round(budget / 1e9, 0) == GOLD["serving_budget_gb"]["value"]
    for ctx, hyb, allm in GOLD["concurrency"]["rows"]:
        assert ca.concurrency(budget, ctx, True) == hyb, ctx
        assert ca.concurrency(budget, ctx, False) == allm, ctx


def test_layer_pattern():
    mla = [i for i in range(72) if ca.mla_layer_index(i)]
    assert mla == GOLD["mla_layers"]["value"]
    assert 72 - len(mla) == ca.HybridShape().kda_layers


def test_mtp_sequence():
    b = ca.per_token_bytes_hybrid(with_mtp=True) * 1_048_576
    assert _round(b / 2**30, 2) == GOLD["mtp_sequence_gib"]["value"]


def test_hybrid_slice_cache():
    # an 8-sequence, 1M-token MLA layer: 8 x 1e6 x 1152 B = 9.216 GB
    assert ca.mla_cache_bytes(8, 1_000_000) == 9_216_000_000
