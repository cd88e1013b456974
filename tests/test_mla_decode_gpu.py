"""Parity of mla_latent_decode (CUDA through the C ABI) with the fp64 oracle.

Scores and softmax are fp32 in the kernel with bf16 tensor-core operands; q and the cache are
bf16 on both sides, so the only extra rounding is P in bf16 for the value contraction. Outputs are
compared as fp32 (LAD_FLAG_OUT_FP32) against the fp64 oracle, and as bf16 against the oracle
rounded to bf16, both within the 2e-3 relative-L2 budget.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from tests.parity import TOL_OUT, bf16_round, f64, max_rel_l2, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lad(cuda_device):
    import latent_attention_decode_b200 as m
    return m


def _inputs(B, lens, lmax, seed, dev):
    cfg = wl.MlaDecode("t", B=B, seed=seed)
    q = wl.normal_bf16((B, 64, wl.D_ROW), seed, "q", dev)
    cache = wl.normal_bf16((B, lmax, wl.D_ROW), seed, "cache", dev)
    gate = wl.normal((B, 64), seed, "gate", dev)
    return q, cache, torch.tensor(lens, dtype=torch.int32, device=dev), gate


def _oracle(q, cache, lens, gate, seqs=None, heads=None):
    seqs = list(range(q.shape[0])) if seqs is None else seqs
    heads = list(range(64)) if heads is None else heads
    qs = f64(q[seqs][:, heads])
    bits = wl.bf16_bits(cache[seqs])
    g = None if gate is None else f64(gate[seqs][:, heads])
    return oracle.mla_decode(qs, bits, f64(lens[seqs]).astype(np.int32), g, scale=wl.MLA_SCALE,
                             nthreads=oracle.max_threads())


def _run(lad, q, cache, lens, gate, out_fp32=True):
    lse = torch.empty((q.shape[0], 64), device=q.device, dtype=torch.float32)
    o = lad.mla_latent_decode(q, cache, lens, gate, lse=lse, out_fp32=out_fp32)
    assert lad.lad_device_error() == 0
    return o, lse


def test_ragged_small(lad, cuda_device):
    """Lengths below, at and across the 32-row tile, with a ragged last tile."""
    lens = [1, 31, 32, 33, 100, 257]
    q, cache, L, gate = _inputs(len(lens), lens, 300, 1, cuda_device)
    o_ref, lse_ref = _oracle(q, cache, L, gate)
    o, lse = _run(lad, q, cache, L, gate)
    assert rel_l2(o, o_ref) < TOL_OUT
    np.testing.assert_allclose(f64(lse), lse_ref, rtol=0, atol=2e-4 * np.abs(lse_ref).max())
    o16, _ = _run(lad, q, cache, L, gate, out_fp32=False)
    assert rel_l2(o16, bf16_round(o_ref)) < TOL_OUT


def test_zero_length_and_no_gate(lad, cuda_device):
    lens = [0, 70, 0]
    q, cache, L, _ = _inputs(3, lens, 96, 2, cuda_device)
    o_ref, lse_ref = _oracle(q, cache, L, None)
    o, lse = _run(lad, q, cache, L, None)
    assert torch.count_nonzero(o[0]) == 0 and torch.count_nonzero(o[2]) == 0
    assert torch.isinf(lse[0]).all() and (lse[0] < 0).all()
    assert rel_l2(o[1], o_ref[1]) < TOL_OUT


def test_all_lengths_zero(lad, cuda_device):
    q, cache, L, gate = _inputs(2, [0, 0], 8, 3, cuda_device)
    o, lse = _run(lad, q, cache, L, gate)
    assert torch.count_nonzero(o) == 0 and torch.isinf(lse).all()


def test_many_short_sequences(lad, cuda_device):
    """More sequences than SMs, so a CTA's share spans several sequences (several segments)."""
    rng = np.random.default_rng(4)
    lens = rng.integers(0, 200, size=400).tolist()
    q, cache, L, gate = _inputs(400, lens, 200, 4, cuda_device)
    o_ref, lse_ref = _oracle(q, cache, L, gate)
    o, lse = _run(lad, q, cache, L, gate)
    assert rel_l2(o, o_ref) < TOL_OUT
    fin = np.isfinite(lse_ref)
    np.testing.assert_allclose(f64(lse)[fin], lse_ref[fin], rtol=0, atol=1e-3)
    assert np.all(np.isneginf(f64(lse)[~fin]))


def test_nan_rows_past_length(lad, cuda_device):
    """Rows past a sequence's length (in its last 32-row tile and beyond) may hold NaN: they get
    exactly zero weight and must not reach the output."""
    lens = [45, 64, 1]
    q, cache, L, gate = _inputs(3, lens, 96, 8, cuda_device)
    o_ref, lse_ref = _oracle(q, cache, L, gate)
    for b, n in enumerate(lens):
        cache[b, n:] = float("nan")
    o, lse = _run(lad, q, cache, L, gate)
    assert torch.isfinite(o).all()
    assert rel_l2(o, o_ref) < TOL_OUT
    np.testing.assert_allclose(f64(lse), lse_ref, rtol=0, atol=1e-3)


def test_padded_cache_stride(lad, cuda_device):
    """The cache is a view into a larger allocation (sequence stride > Lmax rows)."""
    q, big, L, gate = _inputs(3, [50, 64, 10], 128, 5, cuda_device)
    cache = big[:, :80]
    o_ref, _ = _oracle(q, cache.contiguous(), L, gate)
    o, _ = _run(lad, q, cache, L, gate)
    assert rel_l2(o, o_ref) < TOL_OUT


def test_outlier_scores_rescale(lad, cuda_device):
    """A late row far above the running max forces the lazy O rescale path."""
    lens = [4000]
    q, cache, L, gate = _inputs(1, lens, 4000, 6, cuda_device)
    cache[0, 3000] = (q[0, 0].float() * 4.0).to(torch.bfloat16)   # head 0 sees a score jump
    cache[0, 3500] = (q[0, 5].float() * 8.0).to(torch.bfloat16)
    o_ref, lse_ref = _oracle(q, cache, L, gate)
    o, lse = _run(lad, q, cache, L, gate)
    assert rel_l2(o, o_ref) < TOL_OUT
    np.testing.assert_allclose(f64(lse), lse_ref, rtol=0, atol=1e-3)


@pytest.mark.slow
def test_decode_b16_full_size_sampled(lad, cuda_device):
    """The 16-sequence workload (contexts uniform in [8192, 131072]) at full size; the oracle
    checks every head of four sequences (the longest, the shortest and two more)."""
    cfg = wl.CONFIGS["mla_decode_b16"]
    inp = wl.mla_inputs(cfg, cuda_device)
    o, lse = _run(lad, inp["q"], inp["cache"], inp["seq_lens"], inp["gate"])
    lens = inp["seq_lens"].cpu().numpy()
    seqs = sorted({int(np.argmax(lens)), int(np.argmin(lens)), 3, 11})
    o_ref, lse_ref = _oracle(inp["q"], inp["cache"], inp["seq_lens"], inp["gate"], seqs=seqs)
    assert rel_l2(o[seqs], o_ref) < TOL_OUT
    assert max_rel_l2(o[seqs], o_ref, 2) < TOL_OUT   # every (sequence, head) on its own
    np.testing.assert_allclose(f64(lse[seqs]), lse_ref, rtol=0, atol=1e-3)


@pytest.mark.slow
def test_million_token_context_sampled(lad, cuda_device):
    """Two sequences of 1,000,000 cached rows (the 8-layer slice's context): four heads of one
    sequence against the oracle, and the softmax mass invariant through lse for the rest."""
    B, Lc = 2, 1_000_000
    q, cache, L, gate = _inputs(B, [Lc, Lc - 17], Lc, 7, cuda_device)
    o, lse = _run(lad, q, cache, L, gate)
    heads = [0, 17, 42, 63]
    o_ref, lse_ref = _oracle(q, cache, L, gate, seqs=[1], heads=heads)
    assert rel_l2(o[1, heads], o_ref[0]) < TOL_OUT
    np.testing.assert_allclose(f64(lse[1, heads]), lse_ref[0], rtol=0, atol=1e-3)


@pytest.mark.slow
def test_hybrid_launch_8x1m_sampled(lad, cuda_device):
    """The 8-layer hybrid step's latent decode exactly as bench.py launches it: 8 sequences of
    1,000,000 cached rows drawn with the bench's seed; every head of the first sequence and eight
    heads (one per head group of each TMEM sub-partition) of the last, against the oracle, each
    (sequence, head) on its own as well as together."""
    cfg = wl.MlaDecode("mla", B=8, seed=1238, fixed_len=1_000_000)
    inp = wl.mla_inputs(cfg, cuda_device)
    o, lse = _run(lad, inp["q"], inp["cache"], inp["seq_lens"], inp["gate"], out_fp32=False)
    for seqs, heads in (([0], list(range(64))), ([7], [0, 9, 18, 27, 36, 45, 54, 63])):
        o_ref, lse_ref = _oracle(inp["q"], inp["cache"], inp["seq_lens"], inp["gate"], seqs=seqs, heads=heads)
        got = o[seqs][:, heads]
        assert rel_l2(got, bf16_round(o_ref)) < TOL_OUT
        assert max_rel_l2(got, bf16_round(o_ref), 2) < TOL_OUT
        np.testing.assert_allclose(f64(lse[seqs][:, heads]), lse_ref, rtol=0, atol=1e-3)
