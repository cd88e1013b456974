"""Parity of the FP8 (E4M3) latent-cache calls (CUDA through the C ABI) with the fp64 oracle.

- mla_latent_decode_fp8 / mla_latent_decode_paged_fp8 against the oracle's attention over the
  dequantised cache (kv_scale * E4M3(code)), ragged lengths over several tiles, rows past the
  length and spare pages holding the NaN code, Lmax not a multiple of the 32-row tile;
- with a power-of-two kv_scale the FP8 kernel (f16 operands) agrees with the bf16 kernel on the
  dequantised cache: the scores are the same exact products (every E4M3 value and every bf16
  query value of normal f16 range is exact in both types, and scaling by 2^k commutes with the
  roundings), so lse agrees to 1e-5; O differs only by P's rounding (f16 against bf16). A slip in
  the on-chip widening or its swizzled layout moves both by orders of magnitude more;
- the RoPE-in-kernel form against the oracle with the query turned;
- mla_cache_append_fp8 writes the oracle's codes bit for bit (contiguous and paged), and an
  append-then-attend engine step;
- the 16-sequence workload at full size, sampled.
Tolerances: relative L2 2e-3 on outputs (the bf16-input budget), lse within 1e-3.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from tests.parity import TOL_OUT, bf16_round, f64, rel_l2

pytestmark = pytest.mark.gpu

NAN_CODE = 0x7F


@pytest.fixture(scope="module")
def lad(cuda_device):
    import latent_attention_decode_b200 as m
    return m


def _inputs(lens, lmax, seed, dev):
    B = len(lens)
    q = wl.normal_bf16((B, 64, wl.D_ROW), seed, "q", dev)
    codes = wl.e4m3_codes((B, lmax, wl.D_ROW), seed, "cache8", dev)
    L = torch.tensor(lens, dtype=torch.int32, device=dev)
    for b, n in enumerate(lens):  # rows past the length hold NaN: they must get no weight
        codes[b, n:] = NAN_CODE
    gate = wl.normal((B, 64), seed, "gate", dev)
    return q, codes, L, gate


def _oracle(q, codes, lens, gate, kv_scale, seqs=None, heads=None):
    seqs = list(range(q.shape[0])) if seqs is None else seqs
    heads = list(range(64)) if heads is None else heads
    g = None if gate is None else f64(gate[seqs][:, heads])
    return oracle.mla_decode_fp8(f64(q[seqs][:, heads]), codes[seqs].cpu().numpy(), kv_scale,
                                 lens[seqs].cpu().numpy(), g, scale=wl.MLA_SCALE, nthreads=oracle.max_threads())


def _run(lad, q, codes, lens, gate, kv_scale, out_fp32=True):
    lse = torch.empty((q.shape[0], 64), device=q.device, dtype=torch.float32)
    o = lad.mla_latent_decode_fp8(q, codes, kv_scale, lens, gate, lse=lse, out_fp32=out_fp32)
    assert lad.lad_device_error() == 0
    return o, lse


def _check(o, lse, o_ref, lse_ref):
    assert rel_l2(o, o_ref) < TOL_OUT
    fin = np.isfinite(lse_ref)
    np.testing.assert_allclose(f64(lse)[fin], lse_ref[fin], rtol=0, atol=1e-3)
    assert np.all(np.isneginf(f64(lse)[~fin]))


def test_ragged_lengths(lad, cuda_device):
    lens = [1, 31, 32, 33, 100, 291, 0, 64]
    q, codes, L, gate = _inputs(lens, 291, 21, cuda_device)  # Lmax = 291: the last tile is cut by Lmax
    o, lse = _run(lad, q, codes, L, gate, wl.KV_SCALE_FP8)
    assert torch.isfinite(o).all()
    o_ref, lse_ref = _oracle(q, codes, L, gate, wl.KV_SCALE_FP8)
    _check(o, lse, o_ref, lse_ref)
    o16, _ = _run(lad, q, codes, L, gate, wl.KV_SCALE_FP8, out_fp32=False)
    assert rel_l2(o16, bf16_round(o_ref)) < TOL_OUT


def test_general_scale_and_no_gate(lad, cuda_device):
    lens = [77, 513, 5]
    q, codes, L, _ = _inputs(lens, 520, 22, cuda_device)
    kv_scale = 0.0417
    o, lse = _run(lad, q, codes, L, None, kv_scale)
    o_ref, lse_ref = _oracle(q, codes, L, None, kv_scale)
    _check(o, lse, o_ref, lse_ref)


def test_power_of_two_scale_equals_bf16_kernel(lad, cuda_device):
    lens = [45, 300, 1, 257]
    q, codes, L, gate = _inputs(lens, 300, 23, cuda_device)
    kv_scale = 2.0 ** -5
    deq = (codes.view(torch.float8_e4m3fn).to(torch.float32) * kv_scale).to(torch.bfloat16)
    o8, l8 = _run(lad, q, codes, L, gate, kv_scale)
    ob = torch.empty_like(o8)
    lb = torch.empty_like(l8)
    lad.mla_latent_decode(q, deq, L, gate, o=ob, lse=lb, out_fp32=True)
    np.testing.assert_allclose(f64(l8), f64(lb), rtol=0, atol=1e-5)
    assert rel_l2(o8, ob) < TOL_OUT


def test_many_short_sequences(lad, cuda_device):
    """More sequences than SMs: a CTA's share spans several segments, so the widening warps' load
    cursor crosses sequences two tiles ahead of the conversion, and q is converted per segment."""
    rng = np.random.default_rng(29)
    lens = rng.integers(0, 200, size=400).tolist()
    q, codes, L, gate = _inputs(lens, 200, 29, cuda_device)
    o, lse = _run(lad, q, codes, L, gate, wl.KV_SCALE_FP8)
    o_ref, lse_ref = _oracle(q, codes, L, gate, wl.KV_SCALE_FP8)
    _check(o, lse, o_ref, lse_ref)


def test_all_lengths_zero(lad, cuda_device):
    q, codes, L, gate = _inputs([0, 0, 0], 8, 30, cuda_device)
    o, lse = _run(lad, q, codes, L, gate, wl.KV_SCALE_FP8)
    assert torch.count_nonzero(o) == 0 and torch.isinf(lse).all()


def test_paged_many_sequences_and_bad_entry(lad, cuda_device):
    """300 sequences in one shuffled pool of 32-row pages; then one table entry naming no page:
    its rows read as zeros, device error 0x105, the other sequences unaffected."""
    rng = np.random.default_rng(31)
    lens = rng.integers(0, 400, size=300).tolist()
    q, codes, L, gate = _inputs(lens, 400, 31, cuda_device)
    pool, bt = wl.paginate(codes, L, 32, 31)
    o = lad.mla_latent_decode_paged_fp8(q, pool, wl.KV_SCALE_FP8, bt, L, gate_logits=gate, out_fp32=True)
    assert lad.lad_device_error() == 0
    o_ref, _ = oracle.mla_decode_paged_fp8(f64(q), pool.cpu().numpy(), wl.KV_SCALE_FP8, bt.cpu().numpy(),
                                           L.cpu().numpy(), f64(gate), scale=wl.MLA_SCALE,
                                           nthreads=oracle.max_threads())
    assert rel_l2(o, o_ref) < TOL_OUT
    b0 = int(np.argmax(np.asarray(lens) > 64))  # a sequence with a second page
    bad = bt.clone()
    bad[b0, 1] = pool.shape[0] + 5
    o2 = lad.mla_latent_decode_paged_fp8(q, pool, wl.KV_SCALE_FP8, bad, L, gate_logits=gate, out_fp32=True)
    assert lad.lad_device_error() == 0x105
    keep = [b for b in range(len(lens)) if b != b0]
    assert rel_l2(o2[keep], o_ref[keep]) < TOL_OUT
    assert torch.isfinite(o2[b0]).all()


@pytest.mark.parametrize("page_size", [32, 128])
def test_paged_scattered_pages(lad, cuda_device, page_size):
    lens = [1, 31, 33, 257, 0, 64, 200]
    q, codes, L, gate = _inputs(lens, 257, 24, cuda_device)
    pool, bt = wl.paginate(codes, L, page_size, 24, spare_pages=3)  # unused rows and spares: NaN code
    lse = torch.empty((len(lens), 64), device=cuda_device, dtype=torch.float32)
    o = lad.mla_latent_decode_paged_fp8(q, pool, wl.KV_SCALE_FP8, bt, L, gate_logits=gate, lse=lse, out_fp32=True)
    assert lad.lad_device_error() == 0
    o_ref, lse_ref = oracle.mla_decode_paged_fp8(f64(q), pool.cpu().numpy(), wl.KV_SCALE_FP8, bt.cpu().numpy(),
                                                 L.cpu().numpy(), f64(gate), scale=wl.MLA_SCALE,
                                                 nthreads=oracle.max_threads())
    _check(o, lse, o_ref, lse_ref)


@pytest.mark.parametrize("interleaved", [False, True])
def test_paged_query_turned_in_kernel(lad, cuda_device, interleaved):
    lens = [40, 300, 129]
    q, codes, L, gate = _inputs(lens, 300, 25, cuda_device)
    pos = torch.tensor([39, 123456, 7_000_000], dtype=torch.int32, device=cuda_device)
    pool, bt = wl.paginate(codes, L, 64, 25, spare_pages=1)
    lse = torch.empty((len(lens), 64), device=cuda_device, dtype=torch.float32)
    o = lad.mla_latent_decode_paged_fp8(q, pool, wl.KV_SCALE_FP8, bt, L, positions=pos, gate_logits=gate, lse=lse,
                                        interleaved=interleaved, out_fp32=True)
    assert lad.lad_device_error() == 0
    o_ref, lse_ref = oracle.mla_decode_paged_fp8(_turned_q(q, pos.cpu().numpy(), interleaved), pool.cpu().numpy(),
                                                 wl.KV_SCALE_FP8, bt.cpu().numpy(), L.cpu().numpy(), f64(gate),
                                                 scale=wl.MLA_SCALE, nthreads=oracle.max_threads())
    _check(o, lse, o_ref, lse_ref)


def _turned_q(q, pos, interleaved=False):
    """The query with its RoPE part turned in fp64 and rounded to bf16 once, as the kernel stages it."""
    qd = f64(q).copy()
    qd[:, :, wl.D_LATENT:] = oracle.rope(qd[:, :, wl.D_LATENT:], np.asarray(pos)[:, None], interleaved=interleaved)
    return (oracle.round_bf16_bits(qd).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("interleaved", [False, True])
def test_append_writes_oracle_codes(lad, cuda_device, interleaved):
    B, P = 5, 64
    c_kv = wl.normal_bf16((B, wl.D_LATENT), 26, "ckv", cuda_device)
    k_pe = wl.normal_bf16((B, wl.D_ROPE), 26, "kpe", cuda_device)
    pos = torch.tensor([0, 63, 64, 1000, 4_000_000], dtype=torch.int32, device=cuda_device)
    kv_scale = 0.0173
    want = oracle.mla_cache_row_fp8(_bits(c_kv), _bits(k_pe), pos.cpu().numpy(), kv_scale, interleaved=interleaved)
    # contiguous cache of 1001 rows per sequence: the last sequence writes row 17 instead of 4,000,000
    cache = torch.full((B, 1001, wl.D_ROW), NAN_CODE, dtype=torch.uint8, device=cuda_device)
    small = pos.clone()
    small[4] = 17
    lad.mla_cache_append_fp8(c_kv, k_pe, small, cache, kv_scale, interleaved=interleaved)
    assert lad.lad_device_error() == 0
    want_small = oracle.mla_cache_row_fp8(_bits(c_kv), _bits(k_pe), small.cpu().numpy(), kv_scale,
                                          interleaved=interleaved)
    got = np.stack([cache[b, int(small[b])].cpu().numpy() for b in range(B)])
    np.testing.assert_array_equal(got, want_small)
    untouched = cache.clone()
    for b in range(B):
        untouched[b, int(small[b])] = NAN_CODE
    assert (untouched == NAN_CODE).all()
    # paged, large positions
    pages_per = [(int(p) // P) + 1 for p in pos.tolist()]
    n_pages = 8
    bt = torch.full((B, max(pages_per)), -1, dtype=torch.int32)
    for b in range(B):
        bt[b, pages_per[b] - 1] = (3 * b + 1) % n_pages
    bt = bt.to(cuda_device)
    pool = torch.full((n_pages, P, wl.D_ROW), NAN_CODE, dtype=torch.uint8, device=cuda_device)
    lad.mla_cache_append_fp8(c_kv, k_pe, pos, pool, kv_scale, block_table=bt, interleaved=interleaved)
    assert lad.lad_device_error() == 0
    got = np.stack([pool[int(bt[b, pages_per[b] - 1]), int(pos[b]) % P].cpu().numpy() for b in range(B)])
    np.testing.assert_array_equal(got, want)


def test_append_then_attend(lad, cuda_device):
    """An engine step on an FP8 paged cache: each sequence's new row is appended at position
    len - 1, then the query (turned in the kernel to the same position) attends over the pool."""
    lens = [65, 1, 200]
    B = len(lens)
    q, codes, L, gate = _inputs(lens, 200, 27, cuda_device)
    pool, bt = wl.paginate(codes, L, 32, 27, spare_pages=2)
    c_kv = wl.normal_bf16((B, wl.D_LATENT), 27, "ckv", cuda_device)
    k_pe = wl.normal_bf16((B, wl.D_ROPE), 27, "kpe", cuda_device)
    pos = (L - 1).to(torch.int32)
    lad.mla_cache_append_fp8(c_kv, k_pe, pos, pool, wl.KV_SCALE_FP8, block_table=bt)
    o = lad.mla_latent_decode_paged_fp8(q, pool, wl.KV_SCALE_FP8, bt, L, positions=pos, gate_logits=gate,
                                        out_fp32=True)
    assert lad.lad_device_error() == 0
    rows = oracle.mla_cache_row_fp8(_bits(c_kv), _bits(k_pe), pos.cpu().numpy(), wl.KV_SCALE_FP8)
    host_pool = pool.cpu().numpy().copy()
    btn = bt.cpu().numpy()
    for b in range(B):
        p = int(pos[b])
        np.testing.assert_array_equal(host_pool[btn[b, p // 32], p % 32], rows[b])
    o_ref, _ = oracle.mla_decode_paged_fp8(_turned_q(q, pos.cpu().numpy()), host_pool, wl.KV_SCALE_FP8, btn, L.cpu().numpy(), f64(gate),
                                           scale=wl.MLA_SCALE, nthreads=oracle.max_threads())
    assert rel_l2(o, o_ref) < TOL_OUT


@pytest.mark.slow
def test_decode_b16_fp8_full_size_sampled(lad, cuda_device):
    """The 16-sequence workload (contexts uniform in [8192, 131072]) with its FP8 cache, as the
    benchmark launches it; every head of three sequences (the longest, the shortest, one more)."""
    cfg = wl.CONFIGS["mla_decode_b16"]
    inp = wl.mla_inputs(cfg, cuda_device)
    codes = wl.mla_fp8_cache(cfg, cuda_device)
    o, lse = _run(lad, inp["q"], codes, inp["seq_lens"], inp["gate"], wl.KV_SCALE_FP8, out_fp32=False)
    lens = inp["seq_lens"].cpu().numpy()
    seqs = sorted({int(np.argmax(lens)), int(np.argmin(lens)), 5})
    o_ref, lse_ref = _oracle(inp["q"], codes, inp["seq_lens"], inp["gate"], wl.KV_SCALE_FP8, seqs=seqs)
    assert rel_l2(o[seqs], bf16_round(o_ref)) < TOL_OUT
    np.testing.assert_allclose(f64(lse[seqs]), lse_ref, rtol=0, atol=1e-3)


def test_query_beyond_f16_range_is_reported(lad, cuda_device):
    """The FP8 path runs the query in f16: a value beyond +-65504 is reported as device error
    0x106 (the call itself returns normally)."""
    lens = [40, 9]
    q, codes, L, gate = _inputs(lens, 40, 28, cuda_device)
    q[1, 5, 100] = 1.0e5
    lad.mla_latent_decode_fp8(q, codes, wl.KV_SCALE_FP8, L, gate, out_fp32=True)
    assert lad.lad_device_error() == 0x106
    q[1, 5, 100] = 60000.0  # inside the range: no report
    lad.mla_latent_decode_fp8(q, codes, wl.KV_SCALE_FP8, L, gate, out_fp32=True)
    assert lad.lad_device_error() == 0
