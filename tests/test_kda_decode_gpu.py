"""Parity of kda_conv_update and kda_decode_step (CUDA, through the C ABI) with the fp64 oracle.

Inputs come from the seeded workload recipes; the oracle sees the same bf16/fp32 values widened
exactly to fp64. Tolerances are in tests/parity.py.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from tests.parity import TOL_OUT, TOL_STATE, bf16_round, f64, max_rel_l2, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lad(cuda_device):
    import latent_attention_decode_b200 as m
    return m


def _scan(lad, inp, out_fp32, dev, scale=1.0, l2=False):
    q, k, v, a, b = (inp[n].to(dev) for n in ("q", "k", "v", "alpha", "beta"))
    S = inp["S0"].to(dev).clone()
    B, T, H, _ = q.shape
    outs = []
    for t in range(T):
        outs.append(lad.kda_decode_step(q[:, t].contiguous(), k[:, t].contiguous(), v[:, t].contiguous(),
                                        a[:, t].contiguous(), b[:, t].contiguous(), S, scale=scale,
                                        out_fp32=out_fp32, l2norm_qk=l2))
    torch.cuda.synchronize()
    return torch.stack(outs, dim=1), S


def _oracle_scan(inp, scale=1.0, l2=False):
    q, k = f64(inp["q"]), f64(inp["k"])
    if l2:
        q, k = oracle.l2norm(q), oracle.l2norm(k)
    return oracle.kda_recurrent(q, k, f64(inp["v"]), f64(inp["alpha"]), f64(inp["beta"]), f64(inp["S0"]),
                                scale=scale, nthreads=oracle.max_threads())


def test_scan_tiny_256_steps(lad, cuda_device):
    """B=1, H=4, 256 tokens from zero state: every o_t and the final state."""
    inp = wl.kda_scan_inputs(wl.CONFIGS["kda_scan_tiny"])
    o_ref, S_ref = _oracle_scan(inp)
    o32, S = _scan(lad, inp, True, cuda_device)
    assert rel_l2(o32, o_ref) < 1e-5
    assert rel_l2(S, S_ref) < TOL_STATE
    o16, _ = _scan(lad, inp, False, cuda_device)
    assert rel_l2(o16, o_ref) < TOL_OUT
    assert rel_l2(o16, bf16_round(o_ref)) < 2e-4


def test_scan_uniform_decay_nonzero_state_scaled(lad, cuda_device):
    """Every channel decays differently (alpha ~ U[0.9,1)), a live initial state, scale != 1."""
    cfg = wl.KdaScan("u", B=2, H=3, T=64, seed=99, state_std=0.02, alpha_mode="uniform")
    inp = wl.kda_scan_inputs(cfg)
    o_ref, S_ref = _oracle_scan(inp, scale=0.125)
    o, S = _scan(lad, inp, True, cuda_device, scale=0.125)
    assert rel_l2(o, o_ref) < 1e-5 and rel_l2(S, S_ref) < TOL_STATE


def test_l2norm_flag(lad, cuda_device):
    """Unnormalised q, k with the in-kernel L2 normalisation."""
    cfg = wl.KdaScan("n", B=1, H=2, T=16, seed=5, state_std=0.02)
    inp = wl.kda_scan_inputs(cfg)
    inp["q"] = wl.normal_bf16(inp["q"].shape, 5, "qraw", std=3.0)
    inp["k"] = wl.normal_bf16(inp["k"].shape, 5, "kraw", std=0.5)
    o_ref, S_ref = _oracle_scan(inp, l2=True)
    o, S = _scan(lad, inp, True, cuda_device, l2=True)
    assert rel_l2(o, o_ref) < 1e-5 and rel_l2(S, S_ref) < TOL_STATE


def test_identity_step_is_exact(lad, cuda_device):
    """alpha = 1, beta = 0 leaves the fp32 state bit-identical."""
    cfg = wl.KdaScan("i", B=2, H=5, T=1, seed=3, state_std=0.02)
    inp = wl.kda_scan_inputs(cfg)
    inp["alpha"] = torch.ones_like(inp["alpha"])
    inp["beta"] = torch.zeros_like(inp["beta"])
    _, S = _scan(lad, inp, True, cuda_device)
    assert torch.equal(S.cpu(), inp["S0"])


def test_unit_key_full_write(lad, cuda_device):
    """||k|| = 1 (normalised in-kernel) and beta = 1: S^T k = v after the step, to fp32 rounding."""
    cfg = wl.KdaScan("w", B=1, H=4, T=1, seed=4, state_std=0.02)
    inp = wl.kda_scan_inputs(cfg)
    inp["beta"] = torch.ones_like(inp["beta"])
    _, S = _scan(lad, inp, True, cuda_device, l2=True)
    k = oracle.l2norm(f64(inp["k"]))[0, 0]
    v = f64(inp["v"])[0, 0]
    Sk = np.einsum("hij,hi->hj", f64(S)[0], k)
    assert np.abs(Sk - v).max() < 1e-5


def test_decode_b64_conv_then_step(lad, cuda_device):
    """The Ling-shape decode step: conv update of q|k|v for 64 sequences, then the KDA step on
    the conv output (L2-normalised in-kernel) for 64 heads, states ~N(0, 0.02)."""
    cfg = wl.CONFIGS["kda_decode_b64"]
    inp = wl.kda_decode_inputs(cfg, cuda_device)
    B, H, d = cfg.B, cfg.H, 128
    x, tail, w = (f64(inp[n]) for n in ("x", "tail", "w"))
    y_ref, tail_ref = oracle.short_conv_step(x, tail, w, None, silu=True)
    y_ref16 = bf16_round(y_ref)   # the interface stores y in bf16
    qr = oracle.l2norm(y_ref16[:, : H * d].reshape(B, 1, H, d))
    kr = oracle.l2norm(y_ref16[:, H * d: 2 * H * d].reshape(B, 1, H, d))
    vr = y_ref16[:, 2 * H * d:].reshape(B, 1, H, d)
    S0 = f64(inp["S"])
    o_ref, S_ref = oracle.kda_recurrent(qr, kr, vr, f64(inp["alpha"])[:, None], f64(inp["beta"])[:, None],
                                        S0, nthreads=oracle.max_threads())

    y = lad.kda_conv_update(inp["x"], inp["tail"], inp["w"], silu=True)
    o = lad.kda_decode_step(y[:, : H * d], y[:, H * d: 2 * H * d], y[:, 2 * H * d:], inp["alpha"], inp["beta"],
                            inp["S"], l2norm_qk=True, out_fp32=True)
    torch.cuda.synchronize()
    assert np.array_equal(f64(inp["tail"]), tail_ref)
    yg = f64(y)
    assert rel_l2(yg, y_ref) < TOL_OUT
    # fp32 arithmetic then one bf16 rounding: at most one bf16 step away from the rounded oracle
    assert np.all(np.abs(yg - y_ref16) <= np.abs(y_ref16) * 2.0 ** -7 + 1e-30)
    assert rel_l2(o, o_ref[:, 0]) < 1e-4
    assert rel_l2(inp["S"], S_ref) < TOL_STATE
    # per head, against the oracle fed the exact bf16 conv output the step consumed (the rounded
    # fp64 conv output above can differ from it by one bf16 step in a few channels, which moves a
    # single head's o by a few 1e-4)
    q2 = oracle.l2norm(yg[:, : H * d].reshape(B, 1, H, d))
    k2 = oracle.l2norm(yg[:, H * d: 2 * H * d].reshape(B, 1, H, d))
    o2, S2 = oracle.kda_recurrent(q2, k2, yg[:, 2 * H * d:].reshape(B, 1, H, d), f64(inp["alpha"])[:, None],
                                  f64(inp["beta"])[:, None], S0, nthreads=oracle.max_threads())
    assert max_rel_l2(o, o2[:, 0], 2) < 1e-4 and max_rel_l2(inp["S"], S2, 2) < TOL_STATE


@pytest.mark.parametrize("B,H", [(1, 1), (3, 7), (256, 64)])
def test_shapes(lad, cuda_device, B, H):
    cfg = wl.KdaDecode("s", B=B, H=H, seed=11 + B)
    inp = wl.kda_decode_inputs(cfg, cuda_device)
    q = wl.unit_sphere_bf16((B, H, 128), 7, "q", cuda_device)
    k = wl.unit_sphere_bf16((B, H, 128), 7, "k", cuda_device)
    v = wl.normal_bf16((B, H, 128), 7, "v", cuda_device)
    sel = [0, B // 2, B - 1]
    S0 = f64(inp["S"][sel])
    o = lad.kda_decode_step(q, k, v, inp["alpha"], inp["beta"], inp["S"], out_fp32=True)
    torch.cuda.synchronize()
    o_ref, S_ref = oracle.kda_recurrent(f64(q[sel])[:, None], f64(k[sel])[:, None], f64(v[sel])[:, None],
                                        f64(inp["alpha"][sel])[:, None], f64(inp["beta"][sel])[:, None], S0,
                                        nthreads=oracle.max_threads())
    assert rel_l2(o[sel], o_ref[:, 0]) < 1e-5
    assert rel_l2(inp["S"][sel], S_ref) < TOL_STATE


def test_empty_batch_is_noop(lad, cuda_device):
    S = torch.zeros((0, 64, 128, 128), device=cuda_device)
    z = torch.zeros((0, 64, 128), device=cuda_device, dtype=torch.bfloat16)
    o = lad.kda_decode_step(z, z, z, torch.zeros((0, 64, 128), device=cuda_device),
                            torch.zeros((0, 64), device=cuda_device), S)
    assert o.shape == (0, 64, 128)


@pytest.mark.parametrize("silu,bias", [(False, False), (True, True)])
def test_conv_variants(lad, cuda_device, silu, bias):
    B, C = 5, 96
    inp = wl.conv_inputs(B, 21, cuda_device, channels=C)
    bvec = wl.normal_bf16((C,), 21, "bias", cuda_device) if bias else None
    y_ref, tail_ref = oracle.short_conv_step(f64(inp["x"]), f64(inp["tail"]), f64(inp["w"]),
                                             None if bvec is None else f64(bvec), silu=silu)
    y = lad.kda_conv_update(inp["x"], inp["tail"], inp["w"], bias=bvec, silu=silu)
    torch.cuda.synchronize()
    assert np.array_equal(f64(inp["tail"]), tail_ref)
    assert rel_l2(y, y_ref) < TOL_OUT
    y16 = bf16_round(y_ref)
    assert np.all(np.abs(f64(y) - y16) <= np.abs(y16) * 2.0 ** -7 + 1e-30)


def test_conv_rejects_bad_width(lad, cuda_device):
    inp = wl.conv_inputs(2, 1, cuda_device, channels=16, width=3)
    with pytest.raises(lad.LadError) as e:
        lad.kda_conv_update(inp["x"], inp["tail"], inp["w"])
    assert e.value.status == -2


def _fused_oracle(inp, H, silu=True, bias=None):
    """Conv (fp64, no bf16 rounding of its output) -> L2 norm -> one recurrent step."""
    B = inp["x"].shape[0]
    d = 128
    y, tail = oracle.short_conv_step(f64(inp["x"]), f64(inp["tail"]), f64(inp["w"]),
                                     None if bias is None else f64(bias), silu=silu)
    q = oracle.l2norm(y[:, : H * d].reshape(B, 1, H, d))
    k = oracle.l2norm(y[:, H * d: 2 * H * d].reshape(B, 1, H, d))
    v = y[:, 2 * H * d:].reshape(B, 1, H, d)
    o, S = oracle.kda_recurrent(q, k, v, f64(inp["alpha"])[:, None], f64(inp["beta"])[:, None], f64(inp["S"]),
                                nthreads=oracle.max_threads())
    return o[:, 0], S, tail


def test_fused_conv_decode_b64(lad, cuda_device):
    """kda_conv_decode_step on the 64 x 64-head layer: conv, L2 norm and the step in one launch."""
    cfg = wl.CONFIGS["kda_decode_b64"]
    inp = wl.kda_decode_inputs(cfg, cuda_device)
    o_ref, S_ref, tail_ref = _fused_oracle(inp, cfg.H)
    o = lad.kda_conv_decode_step(inp["x"], inp["tail"], inp["w"], inp["alpha"], inp["beta"], inp["S"],
                                 out_fp32=True)
    torch.cuda.synchronize()
    assert np.array_equal(f64(inp["tail"]), tail_ref)
    assert rel_l2(o, o_ref) < 1e-4
    assert rel_l2(inp["S"], S_ref) < TOL_STATE
    assert max_rel_l2(o, o_ref, 2) < 1e-4 and max_rel_l2(inp["S"], S_ref, 2) < TOL_STATE


def _slots():
    """Resident CTAs of the single-token kernel: two per SM."""
    return 2 * torch.cuda.get_device_properties(0).multi_processor_count


def test_fused_conv_decode_b8_paired(lad, cuda_device):
    """The hybrid's KDA layer at full size, 8 sequences x 64 heads: 512 heads are more than the
    resident CTAs, so each CTA updates two heads (the second from shared memory). Every element
    of o, the state and the tails against the oracle; the ungated, gated and two-call forms."""
    cfg = wl.KdaDecode("kda_b8", B=8, seed=1238)
    assert _slots() < cfg.B * cfg.H <= 2 * _slots()
    a = wl.kda_decode_inputs(cfg, cuda_device)
    g = {n: t.clone() for n, t in a.items()}
    c = {n: t.clone() for n, t in a.items()}
    orig = {n: f64(t) for n, t in a.items()}
    o_ref, S_ref, tail_ref = _fused_oracle(a, cfg.H)
    o = lad.kda_conv_decode_step(a["x"], a["tail"], a["w"], a["alpha"], a["beta"], a["S"], out_fp32=True)
    gate = wl.normal_bf16((8, 64, 128), 52, "gate", cuda_device, std=2.0)
    og = lad.kda_conv_decode_step_gated(g["x"], g["tail"], g["w"], g["alpha"], g["beta"], g["S"], gate, None,
                                        eps=1e-5, out_fp32=True)
    hd = cfg.H * 128
    y = lad.kda_conv_update(c["x"], c["tail"], c["w"], silu=True)
    o2 = lad.kda_decode_step(y[:, :hd], y[:, hd:2 * hd], y[:, 2 * hd:], c["alpha"], c["beta"], c["S"],
                             l2norm_qk=True, out_fp32=True)
    torch.cuda.synchronize()
    assert np.array_equal(f64(a["tail"]), tail_ref)
    assert rel_l2(o, o_ref) < 1e-4 and max_rel_l2(o, o_ref, 2) < 1e-4
    assert rel_l2(a["S"], S_ref) < TOL_STATE and max_rel_l2(a["S"], S_ref, 2) < TOL_STATE
    want_g = oracle.gated_rmsnorm(o_ref, f64(gate), None, eps=1e-5)
    assert max_rel_l2(og, want_g, 2) < 1e-4 and torch.equal(g["S"], a["S"])
    # the two-call path's step consumes the conv output as stored (bf16): the oracle of that, per head
    y16 = f64(y)
    qr = oracle.l2norm(y16[:, :hd].reshape(8, 1, 64, 128))
    kr = oracle.l2norm(y16[:, hd:2 * hd].reshape(8, 1, 64, 128))
    o2_ref, S2_ref = oracle.kda_recurrent(qr, kr, y16[:, 2 * hd:].reshape(8, 1, 64, 128), orig["alpha"][:, None],
                                          orig["beta"][:, None], orig["S"], nthreads=oracle.max_threads())
    assert max_rel_l2(o2, o2_ref[:, 0], 2) < 1e-4 and max_rel_l2(c["S"], S2_ref, 2) < TOL_STATE


@pytest.mark.parametrize("extra", ["one_past", "half", "all_paired", "one_more_than_paired"])
def test_paired_launch_boundaries(lad, cuda_device, extra):
    """Head counts around the switch between one and two heads per CTA (one head per sequence so
    that any count is reachable): just above the resident CTAs, in between, exactly twice (every
    CTA paired), and one more (back to one head per CTA)."""
    n = _slots()
    B = {"one_past": n + 1, "half": n + n // 2 + 1, "all_paired": 2 * n, "one_more_than_paired": 2 * n + 1}[extra]
    cfg = wl.KdaDecode("pb", B=B, H=1, seed=60)
    inp = wl.kda_decode_inputs(cfg, cuda_device)
    q = wl.unit_sphere_bf16((B, 1, 128), 61, "q", cuda_device)
    k = wl.unit_sphere_bf16((B, 1, 128), 61, "k", cuda_device)
    v = wl.normal_bf16((B, 1, 128), 61, "v", cuda_device)
    S0 = f64(inp["S"])
    o = lad.kda_decode_step(q, k, v, inp["alpha"], inp["beta"], inp["S"], out_fp32=True)
    torch.cuda.synchronize()
    o_ref, S_ref = oracle.kda_recurrent(f64(q)[:, None], f64(k)[:, None], f64(v)[:, None],
                                        f64(inp["alpha"])[:, None], f64(inp["beta"])[:, None], S0,
                                        nthreads=oracle.max_threads())
    assert max_rel_l2(o, o_ref[:, 0], 2) < 1e-5
    assert max_rel_l2(inp["S"], S_ref, 2) < TOL_STATE


@pytest.mark.parametrize("B,H,silu,bias", [(1, 1, True, False), (3, 5, False, True)])
def test_fused_conv_decode_variants(lad, cuda_device, B, H, silu, bias):
    cfg = wl.KdaDecode("f", B=B, H=H, seed=31 + B)
    inp = wl.kda_decode_inputs(cfg, cuda_device)
    bvec = wl.normal_bf16((3 * H * 128,), 31, "bias", cuda_device) if bias else None
    o_ref, S_ref, tail_ref = _fused_oracle(inp, H, silu=silu, bias=bvec)
    o = lad.kda_conv_decode_step(inp["x"], inp["tail"], inp["w"], inp["alpha"], inp["beta"], inp["S"],
                                 conv_bias=bvec, silu=silu, out_fp32=True)
    torch.cuda.synchronize()
    assert np.array_equal(f64(inp["tail"]), tail_ref)
    assert rel_l2(o, o_ref) < 1e-4 and rel_l2(inp["S"], S_ref) < TOL_STATE


def test_fused_matches_two_calls(lad, cuda_device):
    """The fused path keeps the conv output in fp32; the two-call path stores it as bf16. The two
    kernels must differ by exactly what that rounding does in the oracle."""
    cfg = wl.KdaDecode("t", B=8, seed=41)
    a = wl.kda_decode_inputs(cfg, cuda_device)
    b = {n: t.clone() for n, t in a.items()}
    H, hd = cfg.H, cfg.H * 128
    o_f, _, _ = _fused_oracle(a, H)
    y, _ = oracle.short_conv_step(f64(a["x"]), f64(a["tail"]), f64(a["w"]), None, silu=True)
    y16 = bf16_round(y)
    o_2, _ = oracle.kda_recurrent(oracle.l2norm(y16[:, :hd].reshape(8, 1, H, 128)),
                                  oracle.l2norm(y16[:, hd:2 * hd].reshape(8, 1, H, 128)),
                                  y16[:, 2 * hd:].reshape(8, 1, H, 128), f64(a["alpha"])[:, None],
                                  f64(a["beta"])[:, None], f64(a["S"]), nthreads=oracle.max_threads())
    o1 = lad.kda_conv_decode_step(a["x"], a["tail"], a["w"], a["alpha"], a["beta"], a["S"], out_fp32=True)
    yk = lad.kda_conv_update(b["x"], b["tail"], b["w"], silu=True)
    o2 = lad.kda_decode_step(yk[:, :hd], yk[:, hd:2 * hd], yk[:, 2 * hd:], b["alpha"], b["beta"], b["S"],
                             l2norm_qk=True, out_fp32=True)
    torch.cuda.synchronize()
    assert torch.equal(a["tail"], b["tail"])
    expected = rel_l2(o_2[:, 0], o_f)  # the effect of the bf16 conv output alone
    assert abs(rel_l2(o2, o1) - expected) < 0.05 * expected


@pytest.mark.parametrize("B,H,with_w", [(64, 64, True), (3, 5, False)])
def test_fused_gated_output(lad, cuda_device, B, H, with_w):
    """kda_conv_decode_step_gated: the output gate (gated RMSNorm over each head's 128 outputs)
    fused into the step; the state and tails are those of the ungated call, bit for bit."""
    cfg = wl.KdaDecode("gate", B=B, H=H, seed=50 + B)
    a = wl.kda_decode_inputs(cfg, cuda_device)
    b = {n: t.clone() for n, t in a.items()}
    gate = wl.normal_bf16((B, H, 128), 50, "gate", cuda_device, std=2.0)
    w = (wl.normal((128,), 50, "normw", cuda_device) * 0.2 + 1.0) if with_w else None
    o_ref, S_ref, tail_ref = _fused_oracle(a, H)
    want = oracle.gated_rmsnorm(o_ref, f64(gate), None if w is None else f64(w), eps=1e-5)
    o = lad.kda_conv_decode_step_gated(a["x"], a["tail"], a["w"], a["alpha"], a["beta"], a["S"], gate, w,
                                       eps=1e-5, out_fp32=True)
    lad.kda_conv_decode_step(b["x"], b["tail"], b["w"], b["alpha"], b["beta"], b["S"], out_fp32=True)
    torch.cuda.synchronize()
    assert rel_l2(o, want) < 1e-4
    assert torch.equal(a["S"], b["S"]) and torch.equal(a["tail"], b["tail"])
    assert np.array_equal(f64(a["tail"]), tail_ref) and rel_l2(a["S"], S_ref) < TOL_STATE
    o16 = lad.kda_conv_decode_step_gated(b["x"], b["tail"], b["w"], b["alpha"], b["beta"], b["S"].clone(), gate, w)
    assert o16.dtype == torch.bfloat16


@pytest.mark.parametrize("B", [8, 64])
def test_overlap_prev_chain(lad, cuda_device, B):
    """LAD_FLAG_OVERLAP_PREV: layers launched back to back as programmatic dependents give the
    results of plain launches bit for bit (B = 8 runs the paired kernel, B = 64 one head a CTA).
    Each layer's alpha is the fp32 output of the layer before it, so a read of the inputs before
    the previous kernel has finished would see stale values; the unfused form's step follows the
    conv that writes its q, k, v. The first layer is also checked against the oracle."""
    n = 4
    layers = [wl.kda_decode_inputs(wl.KdaDecode(f"ov{j}", B=B, seed=70 + j), cuda_device) for j in range(n)]
    gate = wl.normal_bf16((B, 64, 128), 79, "gate", cuda_device, std=2.0)
    hd = 64 * 128
    o_ref, S_ref, tail_ref = _fused_oracle(layers[0], 64)

    def run(overlap):
        ls = [{k: t.clone() for k, t in L.items()} for L in layers]
        outs = [torch.empty((B, 64, 128), device=cuda_device, dtype=torch.float32) for _ in range(n)]
        for j, L in enumerate(ls):
            alpha = L["alpha"] if j == 0 else outs[j - 1]
            if j == 2:
                lad.kda_conv_decode_step_gated(L["x"], L["tail"], L["w"], alpha, L["beta"], L["S"], gate, None,
                                               eps=1e-5, o=outs[j], out_fp32=True, overlap_prev=overlap)
            elif j == 3:
                y = lad.kda_conv_update(L["x"], L["tail"], L["w"], silu=True)
                lad.kda_decode_step(y[:, :hd], y[:, hd:2 * hd], y[:, 2 * hd:], alpha, L["beta"], L["S"], o=outs[j],
                                    l2norm_qk=True, out_fp32=True, overlap_prev=overlap)
            else:
                lad.kda_conv_decode_step(L["x"], L["tail"], L["w"], alpha, L["beta"], L["S"], o=outs[j],
                                         out_fp32=True, overlap_prev=overlap)
        torch.cuda.synchronize()
        return ls, outs

    ls0, outs0 = run(False)
    ls1, outs1 = run(True)
    for j in range(n):
        assert torch.equal(outs0[j], outs1[j]), j
        assert torch.equal(ls0[j]["S"], ls1[j]["S"]) and torch.equal(ls0[j]["tail"], ls1[j]["tail"]), j
    assert np.array_equal(f64(ls1[0]["tail"]), tail_ref)
    assert max_rel_l2(outs1[0], o_ref, 2) < 1e-4 and max_rel_l2(ls1[0]["S"], S_ref, 2) < TOL_STATE
