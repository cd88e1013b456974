"""Failure handling without a fault: a barrier wait that can never complete gives up after the
bounded-wait limit, records its tag, raises the CTA's abort flag so that the CTA's other wait
returns at once, and the kernel returns; the context then still runs the kernels (a latent decode
call against the oracle) and the error word reads clean again."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from tests.parity import TOL_OUT, f64, rel_l2

pytestmark = pytest.mark.gpu


def test_wait_that_cannot_complete_gives_up(cuda_device):
    import latent_attention_decode_b200 as lad
    tag, (ok0, ok1, waited_ms, abort) = lad.lad_check_bounded_wait()
    assert tag == 0x401
    assert ok0 == 0 and ok1 == 0 and abort == 1
    assert 300 <= waited_ms <= 900  # returned on warp 0's flag, about half a limit after it started
    # the context is still usable
    q = wl.normal_bf16((2, 64, wl.D_ROW), 31, "q", cuda_device)
    cache = wl.normal_bf16((2, 70, wl.D_ROW), 31, "cache", cuda_device)
    L = torch.tensor([70, 33], dtype=torch.int32, device=cuda_device)
    o = lad.mla_latent_decode(q, cache, L, None, out_fp32=True)
    assert lad.lad_device_error() == 0
    o_ref, _ = oracle.mla_decode(f64(q), wl.bf16_bits(cache), np.array([70, 33], np.int32), None,
                                 scale=wl.MLA_SCALE)
    assert rel_l2(o, o_ref) < TOL_OUT
