"""Parity of kda_decode_multi (T tokens per state pass, CUDA through the C ABI) with the fp64
token-by-token oracle, including the verify-then-commit use (keep the state, then apply only
the accepted prefix). Tolerances as for kda_decode_step (tests/parity.py)."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from tests.parity import TOL_OUT, TOL_STATE, bf16_round, f64, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lad(cuda_device):
    import latent_attention_decode_b200 as m
    return m


def _dev(inp, dev):
    return {n: t.to(dev) for n, t in inp.items()}


def _oracle(inp, scale=1.0, l2=False, T=None):
    sl = slice(None) if T is None else slice(0, T)
    q, k = f64(inp["q"][:, sl]), f64(inp["k"][:, sl])
    if l2:
        q, k = oracle.l2norm(q), oracle.l2norm(k)
    return oracle.kda_recurrent(q, k, f64(inp["v"][:, sl]), f64(inp["alpha"][:, sl]), f64(inp["beta"][:, sl]),
                                f64(inp["S0"]), scale=scale, nthreads=oracle.max_threads())


def _call(lad, d, S, **kw):
    return lad.kda_decode_multi(d["q"], d["k"], d["v"], d["alpha"], d["beta"], S, **kw)


@pytest.mark.parametrize("T,alpha_mode", [(1, "clamped"), (4, "clamped"), (4, "uniform"), (3, "uniform"),
                                          (8, "uniform")])
def test_tokens_per_pass(lad, cuda_device, T, alpha_mode):
    cfg = wl.KdaScan("m", B=3, H=5, T=T, seed=40 + T, state_std=0.02, alpha_mode=alpha_mode)
    inp = wl.kda_scan_inputs(cfg)
    o_ref, S_ref = _oracle(inp, scale=0.5)
    d = _dev(inp, cuda_device)
    S = d["S0"].clone()
    o = _call(lad, d, S, scale=0.5, out_fp32=True)
    assert rel_l2(o, o_ref) < 1e-5
    assert rel_l2(S, S_ref) < TOL_STATE
    S16 = d["S0"].clone()
    o16 = _call(lad, d, S16, scale=0.5)
    assert rel_l2(o16, bf16_round(o_ref)) < 2e-4 and rel_l2(o16, o_ref) < TOL_OUT
    assert torch.equal(S16, S)


def test_strong_decays_lazy_and_eager(lad, cuda_device):
    """The kernel applies a head's decays lazily (the registers hold the state divided by the
    running decay product L of each row; the final state is multiplied back) unless L falls below
    1e-20 on some row, where it decays the state token by token instead. Head 0 keeps the usual
    decays, head 1 decays by 1e-4 a token on some rows (L reaches 1e-16: the lazy form with
    1 / L = 1e16), head 2 by 1e-7 (L reaches 1e-28: the eager form); all three against the oracle."""
    cfg = wl.KdaScan("sd", B=2, H=3, T=4, seed=46, state_std=0.02, alpha_mode="uniform")
    inp = wl.kda_scan_inputs(cfg)
    inp["alpha"][:, :, 1, :32] = 1e-4
    inp["alpha"][:, :, 2, 64:96] = 1e-7
    o_ref, S_ref = _oracle(inp)
    d = _dev(inp, cuda_device)
    S = d["S0"].clone()
    o = _call(lad, d, S, out_fp32=True)
    torch.cuda.synchronize()
    for h in range(3):
        assert rel_l2(o[:, :, h], o_ref[:, :, h]) < 1e-5, h
        assert rel_l2(S[:, h], S_ref[:, h]) < TOL_STATE, h


def test_one_token_equals_decode_step(lad, cuda_device):
    """T = 1 is kda_decode_step up to the fp32 summation order of the column sums."""
    cfg = wl.KdaScan("one", B=4, H=6, T=1, seed=50, state_std=0.02, alpha_mode="uniform")
    d = _dev(wl.kda_scan_inputs(cfg), cuda_device)
    S1, S2 = d["S0"].clone(), d["S0"].clone()
    o1 = _call(lad, d, S1, out_fp32=True)
    o2 = lad.kda_decode_step(d["q"][:, 0].contiguous(), d["k"][:, 0].contiguous(), d["v"][:, 0].contiguous(),
                             d["alpha"][:, 0].contiguous(), d["beta"][:, 0].contiguous(), S2, out_fp32=True)
    assert rel_l2(o1[:, 0], o2) < 1e-6
    assert rel_l2(S1, S2) < 1e-6


def test_l2norm_flag(lad, cuda_device):
    cfg = wl.KdaScan("n", B=2, H=3, T=4, seed=51, state_std=0.02)
    inp = wl.kda_scan_inputs(cfg)
    inp["q"] = wl.normal_bf16(inp["q"].shape, 51, "qraw", std=3.0)
    inp["k"] = wl.normal_bf16(inp["k"].shape, 51, "kraw", std=0.5)
    o_ref, S_ref = _oracle(inp, l2=True)
    d = _dev(inp, cuda_device)
    S = d["S0"].clone()
    o = _call(lad, d, S, l2norm_qk=True, out_fp32=True)
    assert rel_l2(o, o_ref) < 1e-5 and rel_l2(S, S_ref) < TOL_STATE


def test_prefix_lengths_and_untouched_outputs(lad, cuda_device):
    """n_tokens = [0, 2, 4]: sequence 0 keeps its state bit for bit, sequence 1 applies two
    tokens, and output positions past n_b keep what was there."""
    cfg = wl.KdaScan("p", B=3, H=4, T=4, seed=52, state_std=0.02, alpha_mode="uniform")
    inp = wl.kda_scan_inputs(cfg)
    d = _dev(inp, cuda_device)
    S = d["S0"].clone()
    n = torch.tensor([0, 2, 4], dtype=torch.int32, device=cuda_device)
    o = torch.full((3, 4, 4, 128), 7.0, device=cuda_device)
    _call(lad, d, S, o=o, n_tokens=n, out_fp32=True)
    assert torch.equal(S[0], d["S0"][0])
    assert (o[0] == 7.0).all() and (o[1, 2:] == 7.0).all()
    for b, nb in ((1, 2), (2, 4)):
        sub = {k: v[b:b + 1] for k, v in inp.items()}
        o_ref, S_ref = _oracle(sub, T=nb)
        assert rel_l2(o[b:b + 1, :nb], o_ref) < 1e-5
        assert rel_l2(S[b:b + 1], S_ref) < TOL_STATE


def test_verify_then_commit(lad, cuda_device):
    """Speculative cycle: a verify pass with the state kept (outputs for 1 + 3 drafts), then a
    commit of the accepted prefix with no outputs. Equals the oracle on the accepted tokens."""
    cfg = wl.KdaScan("v", B=4, H=8, T=4, seed=53, state_std=0.02)
    inp = wl.kda_scan_inputs(cfg)
    d = _dev(inp, cuda_device)
    S = d["S0"].clone()
    o = _call(lad, d, S, keep_state=True, out_fp32=True)
    assert torch.equal(S, d["S0"])
    o_ref, _ = _oracle(inp)
    assert rel_l2(o, o_ref) < 1e-5
    accepted = torch.tensor([1, 4, 2, 3], dtype=torch.int32, device=cuda_device)
    assert _call(lad, d, S, n_tokens=accepted, want_output=False) is None
    for b, nb in enumerate(accepted.tolist()):
        sub = {k: v[b:b + 1] for k, v in inp.items()}
        _, S_ref = _oracle(sub, T=nb)
        assert rel_l2(S[b:b + 1], S_ref) < TOL_STATE


def test_full_size_b64_four_tokens(lad, cuda_device):
    """64 sequences x 64 heads x 4 tokens (one token plus three drafts), every head."""
    cfg = wl.KdaScan("f", B=64, H=64, T=4, seed=54, state_std=0.02)
    inp = wl.kda_scan_inputs(cfg)
    o_ref, S_ref = _oracle(inp)
    d = _dev(inp, cuda_device)
    S = d["S0"].clone()
    o = _call(lad, d, S)
    assert rel_l2(o, o_ref) < TOL_OUT and rel_l2(o, bf16_round(o_ref)) < 2e-4
    assert rel_l2(S, S_ref) < TOL_STATE


def test_host_checks(lad, cuda_device):
    cfg = wl.KdaScan("h", B=1, H=1, T=9, seed=55, state_std=0.02)
    d = _dev(wl.kda_scan_inputs(cfg), cuda_device)
    with pytest.raises(lad.LadError, match="at most 8"):
        _call(lad, d, d["S0"].clone())
