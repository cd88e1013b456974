"""RoPE applied in the kernels (CUDA through the C ABI) against the fp64 oracle:
- mla_cache_append writes [latent ; RoPE key turned to the position] rows, bit for bit the oracle's
  rows (the rotation is fp64 on both sides and each value is rounded to bf16 once; a value lying
  within ~1e-16 of a rounding boundary may differ by one bf16 step, which the test tolerates in at
  most 1e-4 of the values), into a page pool or the contiguous cache;
- mla_latent_decode_paged_rope turns q's RoPE part to the query position inside the kernel; the
  oracle turns it in fp64 and rounds it to bf16, then attends (tolerance as for the other calls);
- an engine-style step: append every sequence's new row, then attend at position len - 1."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from tests.parity import TOL_OUT, f64, rel_l2

pytestmark = pytest.mark.gpu
THETA = 6.0e6


@pytest.fixture(scope="module")
def lad(cuda_device):
    import latent_attention_decode_b200 as m
    return m


def _bits(t):
    return wl.bf16_bits(t)


def _close_bits(got, want):
    got, want = np.asarray(got, np.int32), np.asarray(want, np.int32)
    diff = np.abs(got - want)
    assert diff.max() <= 1, diff.max()
    assert np.count_nonzero(diff) <= max(1, int(1e-4 * diff.size))


@pytest.mark.parametrize("interleaved", [False, True])
def test_append_paged_rows(lad, cuda_device, interleaved):
    B, P = 5, 64
    lens = torch.tensor([1, 64, 65, 300, 1000], dtype=torch.int32)
    cache = wl.normal_bf16((B, 1024, wl.D_ROW), 21, "cache", cuda_device)
    pool, bt = wl.paginate(cache, torch.tensor([1024] * B, dtype=torch.int32), P, 21)
    before = pool.clone()
    c_kv = wl.normal_bf16((B, 512), 21, "ckv", cuda_device)
    k_pe = wl.normal_bf16((B, 64), 21, "kpe", cuda_device)
    pos = (lens - 1).to(cuda_device)
    lad.mla_cache_append(c_kv, k_pe, pos, pool, block_table=bt, interleaved=interleaved)
    assert lad.lad_device_error() == 0
    want = oracle.mla_cache_row(_bits(c_kv), _bits(k_pe), pos.cpu().numpy(), THETA, interleaved)
    rows = []
    for b in range(B):
        p = int(pos[b])
        rows.append(pool[int(bt[b, p // P]), p % P])
    _close_bits(_bits(torch.stack(rows)), want)
    # nothing else changed
    for b in range(B):
        p = int(pos[b])
        pool[int(bt[b, p // P]), p % P] = before[int(bt[b, p // P]), p % P]
    assert torch.equal(pool.view(torch.int16), before.view(torch.int16))


def test_append_contiguous_large_positions(lad, cuda_device):
    B, L = 3, 4096
    cache = torch.zeros((B, L, wl.D_ROW), dtype=torch.bfloat16, device=cuda_device)
    c_kv = wl.normal_bf16((B, 512), 22, "ckv", cuda_device)
    k_pe = wl.normal_bf16((B, 64), 22, "kpe", cuda_device)
    pos = torch.tensor([0, 17, 4095], dtype=torch.int32, device=cuda_device)
    lad.mla_cache_append(c_kv, k_pe, pos, cache)
    want = oracle.mla_cache_row(_bits(c_kv), _bits(k_pe), pos.cpu().numpy(), THETA)
    got = torch.stack([cache[b, int(pos[b])] for b in range(B)])
    _close_bits(_bits(got), want)
    assert torch.equal(got[0, 512:], k_pe[0])   # position 0 stores the key unchanged
    # large positions through the paged path (one page per sequence, any position inside it)
    pool = torch.zeros((3, 64, wl.D_ROW), dtype=torch.bfloat16, device=cuda_device)
    big = torch.tensor([999_999, 262_143, 123_456], dtype=torch.int32, device=cuda_device)
    bt = torch.full((3, 16384), -1, dtype=torch.int32, device=cuda_device)
    for b in range(3):
        bt[b, int(big[b]) // 64] = b
    lad.mla_cache_append(c_kv, k_pe, big, pool, block_table=bt)
    want = oracle.mla_cache_row(_bits(c_kv), _bits(k_pe), big.cpu().numpy(), THETA)
    got = torch.stack([pool[b, int(big[b]) % 64] for b in range(3)])
    _close_bits(_bits(got), want)


def test_append_position_without_row_is_reported(lad, cuda_device):
    pool = torch.zeros((2, 32, wl.D_ROW), dtype=torch.bfloat16, device=cuda_device)
    bt = torch.tensor([[0], [5]], dtype=torch.int32, device=cuda_device)   # page 5 is not in the pool
    c_kv = wl.normal_bf16((2, 512), 23, "ckv", cuda_device)
    k_pe = wl.normal_bf16((2, 64), 23, "kpe", cuda_device)
    lad.mla_cache_append(c_kv, k_pe, torch.tensor([3, 4], dtype=torch.int32, device=cuda_device), pool,
                         block_table=bt)
    assert lad.lad_device_error() == 0x301
    assert torch.equal(pool[0, 3, :512], c_kv[0]) and torch.count_nonzero(pool[1]) == 0


def _turned_q(q, pos, interleaved):
    """q with its RoPE part turned in fp64 and rounded to bf16 (what the kernel feeds its MMA)."""
    qd = f64(q).copy()
    qd[:, :, 512:] = oracle.rope(qd[:, :, 512:], np.asarray(pos)[:, None], THETA, interleaved)
    bits = oracle.round_bf16_bits(qd)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


@pytest.mark.parametrize("interleaved", [False, True])
def test_decode_turns_query(lad, cuda_device, interleaved):
    lens = [1, 33, 257, 1000, 64]
    q, cache = (wl.normal_bf16((5, 64, wl.D_ROW), 24, "q", cuda_device),
                wl.normal_bf16((5, 1000, wl.D_ROW), 24, "cache", cuda_device))
    gate = wl.normal((5, 64), 24, "gate", cuda_device)
    L = torch.tensor(lens, dtype=torch.int32, device=cuda_device)
    pool, bt = wl.paginate(cache, L, 64, 24)
    pos = torch.tensor([0, 32, 999_999, 999, 63], dtype=torch.int32, device=cuda_device)
    lse = torch.empty((5, 64), device=cuda_device)
    o = lad.mla_latent_decode_paged_rope(q, pos, pool, bt, L, gate, lse=lse, interleaved=interleaved, out_fp32=True)
    assert lad.lad_device_error() == 0
    o_ref, lse_ref = oracle.mla_decode_paged(_turned_q(q, pos.cpu().numpy(), interleaved), wl.bf16_bits(pool),
                                             bt.cpu().numpy(), L.cpu().numpy(), f64(gate), scale=wl.MLA_SCALE,
                                             nthreads=oracle.max_threads())
    assert rel_l2(o, o_ref) < TOL_OUT
    np.testing.assert_allclose(f64(lse), lse_ref, rtol=0, atol=1e-3)


def test_position_zero_equals_unturned_call(lad, cuda_device):
    lens = [500, 70]
    q = wl.normal_bf16((2, 64, wl.D_ROW), 25, "q", cuda_device)
    cache = wl.normal_bf16((2, 512, wl.D_ROW), 25, "cache", cuda_device)
    L = torch.tensor(lens, dtype=torch.int32, device=cuda_device)
    pool, bt = wl.paginate(cache, L, 32, 25)
    zero = torch.zeros(2, dtype=torch.int32, device=cuda_device)
    a = lad.mla_latent_decode_paged_rope(q, zero, pool, bt, L, None, out_fp32=True)
    b = lad.mla_latent_decode_paged(q, pool, bt, L, None, out_fp32=True)
    assert torch.equal(a, b)


def test_engine_step_append_then_attend(lad, cuda_device):
    """Each sequence gets its new token's row (latent + turned RoPE key) appended at position len - 1,
    then the query (RoPE part not yet turned) attends over len rows at that position."""
    B, P = 4, 64
    old = [100, 63, 640, 1]
    cache = wl.normal_bf16((B, 1024, wl.D_ROW), 26, "cache", cuda_device)
    L_new = torch.tensor([n + 1 for n in old], dtype=torch.int32, device=cuda_device)
    pool, bt = wl.paginate(cache, L_new, P, 26)
    c_kv = wl.normal_bf16((B, 512), 26, "ckv", cuda_device)
    k_pe = wl.normal_bf16((B, 64), 26, "kpe", cuda_device)
    q = wl.normal_bf16((B, 64, wl.D_ROW), 26, "q", cuda_device)
    pos = L_new - 1
    lad.mla_cache_append(c_kv, k_pe, pos, pool, block_table=bt)
    o = lad.mla_latent_decode_paged_rope(q, pos, pool, bt, L_new, None, out_fp32=True)
    assert lad.lad_device_error() == 0
    # oracle: the same pool with the oracle's new rows, the oracle's turned query
    pool_bits = wl.bf16_bits(pool).copy()
    rows = oracle.mla_cache_row(_bits(c_kv), _bits(k_pe), pos.cpu().numpy(), THETA)
    for b in range(B):
        p = int(pos[b])
        pool_bits[int(bt[b, p // P]), p % P] = rows[b]
    o_ref, _ = oracle.mla_decode_paged(_turned_q(q, pos.cpu().numpy(), False), pool_bits, bt.cpu().numpy(),
                                       L_new.cpu().numpy(), None, scale=wl.MLA_SCALE, nthreads=oracle.max_threads())
    assert rel_l2(o, o_ref) < TOL_OUT
