"""mla_latent_decode_noalloc: the MLA decode entry point for callers that cannot allocate device
memory (a plugin inside a runtime that owns every allocation, or a decode loop where cudaMalloc's
implicit synchronisation is not allowed). Its scratch space is an array compiled into the library,
so it takes no workspace argument.

Checked through the C ABI against mla_latent_decode (the entry point with a caller workspace) on
two calls in a row with different inputs, so stale scratch from the first call cannot leak into
the second. This file is collected last on purpose.
"""
import ctypes

import pytest
import torch

import workloads as wl
from tests.parity import TOL_OUT, rel_l2

pytestmark = pytest.mark.gpu


def _inputs(lens, lmax, seed, dev):
    B = len(lens)
    q = wl.normal_bf16((B, 64, wl.D_ROW), seed, "q", dev)
    cache = wl.normal_bf16((B, lmax, wl.D_ROW), seed, "cache", dev)
    gate = wl.normal((B, 64), seed, "gate", dev)
    return q, cache, torch.tensor(lens, dtype=torch.int32, device=dev), gate


def _noalloc(lib, q, cache, lens, gate, out_fp32):
    f = lib.mla_latent_decode_noalloc
    f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_longlong, ctypes.c_void_p, ctypes.c_void_p,
                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                  ctypes.c_int, ctypes.c_float, ctypes.c_uint, ctypes.c_void_p]
    f.restype = ctypes.c_int
    B = q.shape[0]
    o = torch.empty((B, 64, 512), device=q.device, dtype=torch.float32 if out_fp32 else torch.bfloat16)
    lse = torch.empty((B, 64), device=q.device, dtype=torch.float32)
    rc = f(q.data_ptr(), cache.data_ptr(), cache.stride(0), lens.data_ptr(), gate.data_ptr(), o.data_ptr(),
           lse.data_ptr(), B, 64, 512, 64, cache.shape[1], wl.MLA_SCALE, 4 if out_fp32 else 0,
           torch.cuda.current_stream().cuda_stream)
    assert rc == 0, lib.lad_last_error()
    return o, lse


def test_noalloc_matches_workspace_entry_point(cuda_device):
    import latent_attention_decode_b200 as lad
    cases = [([300, 1, 0, 4097, 33], 4100, 31, True), ([2000] * 3 + [17], 2000, 32, False)]
    for lens, lmax, seed, f32 in cases:  # two calls in a row share the scratch array
        q, cache, L, gate = _inputs(lens, lmax, seed, cuda_device)
        o_n, lse_n = _noalloc(lad._lib, q, cache, L, gate, f32)
        lse_w = torch.empty_like(lse_n)
        o_w = lad.mla_latent_decode(q, cache, L, gate, lse=lse_w, out_fp32=f32)
        torch.cuda.synchronize()
        assert lad.lad_device_error() == 0
        assert rel_l2(o_n, o_w) < TOL_OUT
        fin = torch.isfinite(lse_w)
        assert torch.equal(fin, torch.isfinite(lse_n))
        assert rel_l2(lse_n[fin], lse_w[fin]) < TOL_OUT


def test_noalloc_python_wrapper(cuda_device):
    """The binding's own marshalling (shape checks, the single-sequence stride, d_rope = D - 512)
    with caller-allocated o and lse, including B = 1, against the workspace entry point."""
    import latent_attention_decode_b200 as lad
    for lens, lmax, seed in (([777], 800, 41), ([5, 0, 1200, 64], 1300, 42)):
        q, cache, L, gate = _inputs(lens, lmax, seed, cuda_device)
        B = len(lens)
        o_n = torch.empty((B, 64, 512), device=cuda_device, dtype=torch.float32)
        lse_n = torch.empty((B, 64), device=cuda_device, dtype=torch.float32)
        out = lad.mla_latent_decode_noalloc(q, cache, L, gate, o=o_n, lse=lse_n, out_fp32=True)
        assert out.data_ptr() == o_n.data_ptr()
        lse_w = torch.empty_like(lse_n)
        o_w = lad.mla_latent_decode(q, cache, L, gate, lse=lse_w, out_fp32=True)
        torch.cuda.synchronize()
        assert lad.lad_device_error() == 0
        assert rel_l2(o_n, o_w) < TOL_OUT
        fin = torch.isfinite(lse_w)
        assert torch.equal(fin, torch.isfinite(lse_n))
        assert rel_l2(lse_n[fin], lse_w[fin]) < TOL_OUT


def test_noalloc_rejects_batch_over_limit(cuda_device):
    import latent_attention_decode_b200 as lad
    lim = lad._lib.mla_latent_decode_noalloc_max_batch()
    q, cache, L, gate = _inputs([8] * (lim + 1), 8, 3, cuda_device)
    o = torch.full((lim + 1, 64, 512), 7.0, device=cuda_device, dtype=torch.bfloat16)
    f = lad._lib.mla_latent_decode_noalloc
    rc = f(q.data_ptr(), cache.data_ptr(), cache.stride(0), L.data_ptr(), gate.data_ptr(), o.data_ptr(), None,
           lim + 1, 64, 512, 64, 8, wl.MLA_SCALE, 0, None)
    assert rc == -2 and b"scratch limit" in lad._lib.lad_last_error()
    torch.cuda.synchronize()
    assert bool((o == 7.0).all())  # rejected before any launch: o untouched
