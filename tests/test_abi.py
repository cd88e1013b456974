"""The C-ABI library loads, exports every function include/lad.h declares, and rejects bad
arguments on the host before touching a GPU (these calls launch nothing)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "lad.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*([a-z_][a-z_0-9]*)\s*\(", src, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    from latent_attention_decode_b200 import build
    build.build()
    import latent_attention_decode_b200 as lad
    return lad._lib


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert {"kda_conv_update", "kda_decode_step", "kda_prefill_chunked", "mla_latent_decode",
            "lad_last_error", "mla_latent_decode_workspace_size", "kda_prefill_workspace_size"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_host_side_validation(lib):
    import latent_attention_decode_b200 as lad
    # unsupported head size
    rc = lib.kda_decode_step(1, 1, 1, 0, 1, 1, 16, 16, 1, 1, 64, 64, 1.0, 0, None)
    assert rc == -2 and b"128" in lib.lad_last_error()
    # null pointers
    assert lib.kda_decode_step(None, 1, 1, 0, 1, 1, 16, 16, 1, 1, 128, 128, 1.0, 0, None) == -1
    # empty batch is a no-op
    assert lib.kda_decode_step(None, None, None, 0, None, None, None, None, 0, 64, 128, 128, 1.0, 0, None) == 0
    # conv: width other than 4, channels not a multiple of 8, misaligned pointers, unknown flags
    assert lib.kda_conv_update(16, 16, 16, None, 32, 1, 16, 3, 0, None) == -2
    assert lib.kda_conv_update(16, 16, 16, None, 32, 1, 12, 4, 0, None) == -2
    assert lib.kda_conv_update(18, 16, 16, None, 32, 1, 16, 4, 0, None) == -2
    assert lib.kda_conv_update(16, 16, 16, None, 32, 1, 16, 4, 0x80, None) == -1
    assert lib.kda_conv_update(16, 16, 16, None, 16, 1, 16, 4, 0, None) == -1  # y aliases x
    assert lad.lad_version() >= 100
