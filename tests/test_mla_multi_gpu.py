"""Parity of mla_latent_decode_multi (the MLA half of a multi-token verify step) with the fp64
oracle: token j of sequence b attends the first seq_lens[b] - T + 1 + j cached rows, so the
oracle is the single-token attention over a batch of B*T sequences that repeat each cache T times
with those lengths. T = 1 is the single-token call bit for bit."""
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


def _inputs(lens, T, lmax, seed, dev):
    B = len(lens)
    q = wl.normal_bf16((B, T, 64, wl.D_ROW), seed, "q", dev)
    cache = wl.normal_bf16((B, lmax, wl.D_ROW), seed, "cache", dev)
    gate = wl.normal((B, T, 64), seed, "gate", dev)
    return q, cache, torch.tensor(lens, dtype=torch.int32, device=dev), gate


def _oracle(q, cache, lens, gate):
    B, T = q.shape[0], q.shape[1]
    vl = np.array([max(0, int(lens[b]) - (T - 1 - j)) for b in range(B) for j in range(T)], dtype=np.int32)
    bits = np.repeat(wl.bf16_bits(cache), T, axis=0)
    g = None if gate is None else f64(gate).reshape(B * T, 64)
    o, lse = oracle.mla_decode(f64(q).reshape(B * T, 64, wl.D_ROW), bits, vl, g, scale=wl.MLA_SCALE,
                               nthreads=oracle.max_threads())
    return o.reshape(B, T, 64, -1), lse.reshape(B, T, 64)


def test_one_token_equals_single_token_call(lad, cuda_device):
    lens = [37, 300, 1, 129]
    q, cache, L, gate = _inputs(lens, 1, 300, 41, cuda_device)
    lse1 = torch.empty((4, 1, 64), device=cuda_device)
    o1 = lad.mla_latent_decode_multi(q, cache, L, gate, lse=lse1, out_fp32=True)
    lse0 = torch.empty((4, 64), device=cuda_device)
    o0 = lad.mla_latent_decode(q[:, 0].contiguous(), cache, L, gate[:, 0].contiguous(), lse=lse0, out_fp32=True)
    assert lad.lad_device_error() == 0
    assert torch.equal(o1[:, 0], o0) and torch.equal(lse1[:, 0], lse0)


@pytest.mark.parametrize("T", [2, 4])
def test_tokens_attend_causally(lad, cuda_device, T):
    lens = [1, 3, 33, 260, 64, 0]  # rows include the T tokens' own; some have fewer rows than tokens
    q, cache, L, gate = _inputs(lens, T, 260, 42 + T, cuda_device)
    lse = torch.empty((len(lens), T, 64), device=cuda_device)
    o = lad.mla_latent_decode_multi(q, cache, L, gate, lse=lse, out_fp32=True)
    assert lad.lad_device_error() == 0
    o_ref, lse_ref = _oracle(q, cache, L.cpu().numpy(), gate)
    assert torch.isfinite(o).all()
    assert rel_l2(o, o_ref) < TOL_OUT
    fin = np.isfinite(lse_ref)
    np.testing.assert_allclose(f64(lse)[fin], lse_ref[fin], rtol=0, atol=1e-3)
    assert np.all(np.isneginf(f64(lse)[~fin]))
    o16 = lad.mla_latent_decode_multi(q, cache, L, gate, out_fp32=False)
    assert rel_l2(o16, bf16_round(o_ref)) < TOL_OUT


def test_many_sequences_three_draft_tokens(lad, cuda_device):
    """The pages' three speculative tokens, over more sequences than SMs (several segments per CTA)."""
    rng = np.random.default_rng(43)
    lens = rng.integers(0, 150, size=120).tolist()
    q, cache, L, _ = _inputs(lens, 3, 150, 43, cuda_device)
    o = lad.mla_latent_decode_multi(q, cache, L, None, out_fp32=True)
    assert lad.lad_device_error() == 0
    o_ref, _ = _oracle(q, cache, L.cpu().numpy(), None)
    assert rel_l2(o, o_ref) < TOL_OUT
