"""Parity of mla_latent_decode_paged (CUDA through the C ABI) with the fp64 oracle over a paged
cache: pages scattered through a pool in random order, NaN in every row past a sequence's
length and in spare pages, several page sizes. Tolerances as for the contiguous call."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from tests.parity import TOL_OUT, bf16_round, f64, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lad(cuda_device):
    import latent_attention_decode_b200 as m
    return m


def _inputs(lens, lmax, seed, dev, page_size, spare=3):
    B = len(lens)
    q = wl.normal_bf16((B, 64, wl.D_ROW), seed, "q", dev)
    cache = wl.normal_bf16((B, lmax, wl.D_ROW), seed, "cache", dev)
    gate = wl.normal((B, 64), seed, "gate", dev)
    L = torch.tensor(lens, dtype=torch.int32, device=dev)
    pool, bt = wl.paginate(cache, L, page_size, seed, spare_pages=spare)
    return q, pool, bt, L, gate


def _oracle(q, pool, bt, lens, gate, seqs=None):
    seqs = list(range(q.shape[0])) if seqs is None else seqs
    g = None if gate is None else f64(gate[seqs])
    return oracle.mla_decode_paged(f64(q[seqs]), wl.bf16_bits(pool), bt[seqs].cpu().numpy(),
                                   lens[seqs].cpu().numpy(), g, scale=wl.MLA_SCALE, nthreads=oracle.max_threads())


def _run(lad, q, pool, bt, lens, gate, out_fp32=True):
    lse = torch.empty((q.shape[0], 64), device=q.device, dtype=torch.float32)
    o = lad.mla_latent_decode_paged(q, pool, bt, lens, gate, lse=lse, out_fp32=out_fp32)
    assert lad.lad_device_error() == 0
    return o, lse


@pytest.mark.parametrize("page_size", [32, 64, 256])
def test_ragged_lengths_scattered_pages(lad, cuda_device, page_size):
    lens = [1, 31, 32, 33, 100, 257, 0, 64]
    q, pool, bt, L, gate = _inputs(lens, 300, 11, cuda_device, page_size)
    o_ref, lse_ref = _oracle(q, pool, bt, L, gate)
    o, lse = _run(lad, q, pool, bt, L, gate)
    assert torch.isfinite(o).all()
    assert rel_l2(o, o_ref) < TOL_OUT
    fin = np.isfinite(lse_ref)
    np.testing.assert_allclose(f64(lse)[fin], lse_ref[fin], rtol=0, atol=1e-3)
    assert np.all(np.isneginf(f64(lse)[~fin]))
    o16, _ = _run(lad, q, pool, bt, L, gate, out_fp32=False)
    assert rel_l2(o16, bf16_round(o_ref)) < TOL_OUT


def test_many_sequences_shared_pool(lad, cuda_device):
    """More sequences than SMs; a CTA's share crosses many sequences and page-table refills."""
    rng = np.random.default_rng(12)
    lens = rng.integers(0, 400, size=300).tolist()
    q, pool, bt, L, gate = _inputs(lens, 400, 12, cuda_device, 32, spare=0)
    o_ref, _ = _oracle(q, pool, bt, L, gate)
    o, _ = _run(lad, q, pool, bt, L, gate)
    assert rel_l2(o, o_ref) < TOL_OUT


def test_long_sequence_many_pages(lad, cuda_device):
    """One sequence of 40,000 rows in 64-row pages: 625 table entries, refilled 32 at a time."""
    q, pool, bt, L, gate = _inputs([40_000, 5], 40_000, 13, cuda_device, 64)
    o_ref, lse_ref = _oracle(q, pool, bt, L, gate)
    o, lse = _run(lad, q, pool, bt, L, gate)
    assert rel_l2(o, o_ref) < TOL_OUT
    np.testing.assert_allclose(f64(lse), lse_ref, rtol=0, atol=1e-3)


def test_identity_table_equals_contiguous_call(lad, cuda_device):
    """With pages laid out in order, the paged call reads the same rows as the contiguous call
    on the same memory: both agree with the oracle and with each other to rounding order."""
    lens = [500, 77]
    B, P = 2, 64
    q = wl.normal_bf16((B, 64, wl.D_ROW), 14, "q", cuda_device)
    cache = wl.normal_bf16((B, 512, wl.D_ROW), 14, "cache", cuda_device)
    L = torch.tensor(lens, dtype=torch.int32, device=cuda_device)
    pool = cache.reshape(B * 512 // P, P, wl.D_ROW)
    bt = torch.arange(B * 512 // P, dtype=torch.int32, device=cuda_device).reshape(B, -1)
    o_p, _ = _run(lad, q, pool, bt, L, None)
    o_c = lad.mla_latent_decode(q, cache, L, None, out_fp32=True)
    o_ref, _ = oracle.mla_decode(f64(q), wl.bf16_bits(cache), lens, None, scale=wl.MLA_SCALE,
                                 nthreads=oracle.max_threads())
    assert rel_l2(o_p, o_ref) < TOL_OUT and rel_l2(o_c, o_ref) < TOL_OUT
    assert torch.equal(o_p, o_c)   # same tiles in the same order: the same arithmetic


def test_block_table_entry_outside_pool_is_reported(lad, cuda_device):
    """A needed entry that names no page reads as zeros and sets device error 0x105; the other
    sequences are unaffected."""
    q, pool, bt, L, gate = _inputs([100, 70], 128, 15, cuda_device, 32)
    bad = bt.clone()
    bad[0, 1] = pool.shape[0] + 7
    o = lad.mla_latent_decode_paged(q, pool, bad, L, gate, out_fp32=True)
    assert lad.lad_device_error() == 0x105
    o_ref, _ = _oracle(q, pool, bt, L, gate, seqs=[1])
    assert rel_l2(o[1:], o_ref) < TOL_OUT
    assert lad.lad_device_error() == 0


def test_host_checks(lad, cuda_device):
    q, pool, bt, L, gate = _inputs([10], 32, 16, cuda_device, 32)
    odd = torch.zeros((2, 48, wl.D_ROW), dtype=torch.bfloat16, device=cuda_device)
    with pytest.raises(lad.LadError, match="multiple of 32"):
        lad.mla_latent_decode_paged(q, odd, bt, L, gate)


@pytest.mark.slow
def test_decode_b16_paged_full_size_sampled(lad, cuda_device):
    """The 16-sequence workload in 64-row pages at full size; every head of four sequences
    against the oracle."""
    cfg = wl.CONFIGS["mla_decode_b16"]
    inp = wl.mla_inputs(cfg, cuda_device)
    pool, bt = wl.paginate(inp["cache"], inp["seq_lens"], 64, cfg.seed)
    cache = inp.pop("cache")
    o, lse = _run(lad, inp["q"], pool, bt, inp["seq_lens"], inp["gate"])
    lens = inp["seq_lens"].cpu().numpy()
    seqs = sorted({int(np.argmax(lens)), int(np.argmin(lens)), 3, 11})
    o_ref, lse_ref = oracle.mla_decode(f64(inp["q"][seqs]), wl.bf16_bits(cache[seqs]), lens[seqs],
                                       f64(inp["gate"][seqs]), scale=wl.MLA_SCALE, nthreads=oracle.max_threads())
    assert rel_l2(o[seqs], o_ref) < TOL_OUT
    np.testing.assert_allclose(f64(lse[seqs]), lse_ref, rtol=0, atol=1e-3)
