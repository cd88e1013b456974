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


def test_flag_values_match_the_header(lib):
    import latent_attention_decode_b200 as lad
    src = open(os.path.join(ROOT, "include", "lad.h")).read()
    flags = {m.group(1): int(m.group(2)) for m in re.finditer(r"#define LAD_(FLAG_[A-Z0-9_]+) \(1u << (\d+)\)", src)}
    assert {"FLAG_SILU", "FLAG_OVERLAP_PREV"} <= set(flags)
    for name, bit in flags.items():
        assert getattr(lad, name) == 1 << bit, name
    # the overlap flag belongs to the single-token KDA calls; the multi-token call rejects it
    assert lib.kda_decode_multi(16, 16, 16, 16, 16, 16, None, None, 1, 4, 1, 128, 128, 1.0, lad.FLAG_OVERLAP_PREV,
                                None) == -1


def test_host_side_validation_of_the_newer_calls(lib):
    """Each of these returns before any CUDA call (no GPU here)."""
    # kda_decode_multi: more than 8 tokens, unknown flag, head size, empty work
    assert lib.kda_decode_multi(16, 16, 16, 16, 16, 16, None, None, 1, 9, 1, 128, 128, 1.0, 0, None) == -2
    assert lib.kda_decode_multi(16, 16, 16, 16, 16, 16, None, None, 1, 4, 1, 128, 128, 1.0, 0x100, None) == -1
    assert lib.kda_decode_multi(16, 16, 16, 16, 16, 16, None, None, 1, 4, 1, 64, 64, 1.0, 0, None) == -2
    assert lib.kda_decode_multi(None, None, None, None, None, None, None, None, 0, 4, 1, 128, 128, 1.0, 0, None) == 0
    assert lib.kda_decode_multi(None, 16, 16, 16, 16, 16, None, None, 1, 4, 1, 128, 128, 1.0, 0, None) == -1
    # mla_latent_decode_paged: page size not a multiple of 32, head count, scale
    args = (16, 16, 4, 48, 16, 1, 16, None, 16, None, 1, 64, 512, 64, 0.1, 0, 16, 1 << 20, None)
    assert lib.mla_latent_decode_paged(*args) == -2 and b"multiple of 32" in lib.lad_last_error()
    bad_h = list(args); bad_h[3] = 64; bad_h[11] = 32
    assert lib.mla_latent_decode_paged(*bad_h) == -2
    bad_s = list(args); bad_s[3] = 64; bad_s[14] = -1.0
    assert lib.mla_latent_decode_paged(*bad_s) == -1
    # mla_latent_decode_paged_rope: rope_theta must exceed 1, positions required
    r = (16, 16, 1.0, 16, 4, 64, 16, 1, 16, None, 16, None, 1, 64, 512, 64, 0.1, 0, 16, 1 << 20, None)
    assert lib.mla_latent_decode_paged_rope(*r) == -1 and b"rope_theta" in lib.lad_last_error()
    r2 = list(r); r2[1] = None; r2[2] = 6.0e6
    assert lib.mla_latent_decode_paged_rope(*r2) == -1 and b"positions" in lib.lad_last_error()
    # mla_cache_append: unknown flag, widths, theta, contiguous stride too small, empty batch
    a = [16, 16, 16, 16, 576 * 8, 8, None, 0, 0, 0, 1, 512, 64, 6.0e6, 0, None]
    assert lib.mla_cache_append(*(a[:14] + [0x40] + a[15:])) == -1
    assert lib.mla_cache_append(*(a[:11] + [256] + a[12:])) == -2
    assert lib.mla_cache_append(*(a[:13] + [0.5] + a[14:])) == -1
    assert lib.mla_cache_append(*(a[:4] + [576] + a[5:])) == -1 and b"cache_seq_stride" in lib.lad_last_error()
    assert lib.mla_cache_append(*(a[:10] + [0] + a[11:])) == 0


def test_host_side_validation_of_the_fp8_calls(lib):
    """FP8 cache calls: kv_scale, stride and alignment checks return before any CUDA call."""
    # mla_latent_decode_fp8(q, cache, stride, kv_scale, lens, gate, o, lse, B, Hq, Dl, Dr, Lmax, scale, flags, ws,
    #                       ws_bytes, stream)
    d = [16, 16, 576 * 8, 0.5, 16, None, 16, None, 1, 64, 512, 64, 8, 0.1, 0, 16, 1 << 20, None]
    bad = list(d); bad[3] = 0.0
    assert lib.mla_latent_decode_fp8(*bad) == -1 and b"kv_scale" in lib.lad_last_error()
    bad = list(d); bad[3] = float("inf")
    assert lib.mla_latent_decode_fp8(*bad) == -1
    bad = list(d); bad[2] = 576 * 8 + 8  # bytes between sequences must be a multiple of 16
    assert lib.mla_latent_decode_fp8(*bad) == -1 and b"multiple of 16" in lib.lad_last_error()
    bad = list(d); bad[1] = 24  # the cache must be 16-byte aligned
    assert lib.mla_latent_decode_fp8(*bad) == -2
    bad = list(d); bad[8] = 0
    assert lib.mla_latent_decode_fp8(*bad) == 0
    # mla_latent_decode_paged_fp8(q, positions, theta, pages, kv_scale, num_pages, page_size, bt, bt_stride, lens,
    #                             gate, o, lse, B, Hq, Dl, Dr, scale, flags, ws, ws_bytes, stream)
    p = [16, None, 6.0e6, 16, 0.5, 4, 48, 16, 1, 16, None, 16, None, 1, 64, 512, 64, 0.1, 0, 16, 1 << 20, None]
    assert lib.mla_latent_decode_paged_fp8(*p) == -2 and b"multiple of 32" in lib.lad_last_error()
    bad = list(p); bad[6] = 64; bad[4] = -1.0
    assert lib.mla_latent_decode_paged_fp8(*bad) == -1 and b"kv_scale" in lib.lad_last_error()
    bad = list(p); bad[6] = 64; bad[1] = 16; bad[2] = 0.5
    assert lib.mla_latent_decode_paged_fp8(*bad) == -1 and b"rope_theta" in lib.lad_last_error()
    bad = list(p); bad[6] = 64; bad[18] = 1 << 4  # the interleaved pairing needs positions
    assert lib.mla_latent_decode_paged_fp8(*bad) == -1
    # mla_cache_append_fp8(c_kv, k_pe, positions, cache, stride, Lmax, bt, bt_stride, num_pages, page_size, B, Dl,
    #                      Dr, theta, kv_scale, flags, stream)
    a = [16, 16, 16, 16, 576 * 8, 8, None, 0, 0, 0, 1, 512, 64, 6.0e6, 0.5, 0, None]
    bad = list(a); bad[14] = 0.0
    assert lib.mla_cache_append_fp8(*bad) == -1 and b"kv_scale" in lib.lad_last_error()
    bad = list(a); bad[4] = 576 * 8 + 8
    assert lib.mla_cache_append_fp8(*bad) == -1 and b"multiple of 16" in lib.lad_last_error()
    bad = list(a); bad[10] = 0
    assert lib.mla_cache_append_fp8(*bad) == 0


def test_prefill_workspace_size(lib):
    """The two-kernel prefill path's workspace: a 256-byte header of per-segment item counters,
    then one 74,240-byte record (fp16 / bf16 operand tiles and g_last) per (sequence, head, chunk) of
    a segment of at most 128 chunks, twice over when there are several segments (one segment's
    records are read while the next one's are written); zero for shapes the call does not
    support."""
    rec, hdr = 74240, 256
    assert lib.kda_prefill_workspace_size(1, 32768, 64, 128, 128, 64) == hdr + 2 * 64 * 128 * rec
    assert lib.kda_prefill_workspace_size(1, 128 * 64 + 1, 1, 128, 128, 64) == hdr + 2 * 128 * rec
    assert lib.kda_prefill_workspace_size(1, 128 * 64, 1, 128, 128, 64) == hdr + 128 * rec
    assert lib.kda_prefill_workspace_size(2, 100, 3, 128, 128, 64) == hdr + 2 * 3 * 2 * rec
    assert lib.kda_prefill_workspace_size(1, 1, 1, 128, 128, 64) == hdr + rec
    assert lib.kda_prefill_workspace_size(1, 0, 64, 128, 128, 64) == 0
    assert lib.kda_prefill_workspace_size(1, 64, 64, 64, 128, 64) == 0
    assert lib.kda_prefill_workspace_size(1, 64, 64, 128, 128, 32) == 0


def test_prefill_workspace_given_too_small(lib):
    """A workspace that is given must hold kda_prefill_workspace_size bytes (NULL selects the
    single-kernel path instead); the check comes before any CUDA call."""
    rc = lib.kda_prefill_chunked(16, 16, 16, 16, 16, 16, 16, 1, 64, 1, 128, 128, 64, 1.0, 0, 16, 100, None)
    assert rc == -4 and b"workspace" in lib.lad_last_error()
    rc = lib.kda_prefill_chunked(16, 16, 16, 16, 16, 16, 16, 1, 64, 1, 128, 128, 64, 1.0, 0, 24, 1 << 20, None)
    assert rc == -4  # misaligned


def test_multi_token_mla_host_checks(lib):
    # mla_latent_decode_multi(q, cache, stride, lens, gate, o, lse, B, T, Hq, Dl, Dr, Lmax, scale, flags, ws, ws_bytes,
    #                         stream)
    a = [16, 16, 576 * 8, 16, None, 16, None, 1, 4, 64, 512, 64, 8, 0.1, 0, 16, 1 << 20, None]
    bad = list(a); bad[8] = 0
    assert lib.mla_latent_decode_multi(*bad) == -1 and b"T must be" in lib.lad_last_error()
    bad = list(a); bad[9] = 32
    assert lib.mla_latent_decode_multi(*bad) == -2
    bad = list(a); bad[7] = 0
    assert lib.mla_latent_decode_multi(*bad) == 0
    assert lib.mla_latent_decode_multi_workspace_size(2, 4, 64, 512, 10) == \
        lib.mla_latent_decode_workspace_size(8, 64, 512, 10) + 256
    assert lib.mla_latent_decode_multi_workspace_size(2, 0, 64, 512, 10) == 0


def test_binding_covers_every_declared_call(lib):
    """Every call include/lad.h declares has a Python wrapper of the same name in the binding
    (argument marshalling only), except the error-string accessor and the no-alloc batch limit,
    which the binding uses internally."""
    import latent_attention_decode_b200 as lad
    internal = {"lad_last_error", "mla_latent_decode_noalloc_max_batch"}
    missing = [n for n in _declared() if n not in internal and not callable(getattr(lad, n, None))]
    assert not missing, missing
    for n in lad.__all__:
        assert hasattr(lad, n), n
