"""Plain fp64 CPU oracle for the hybrid-attention decode path.

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py`` are the only callers. The product library never imports this package, and
this package never imports the product library; the two share no code.

The arithmetic lives in ``lad_oracle.c`` (double precision, loops written as the definitions
read). This module compiles it with gcc on first use (or on ``build()``) and wraps each entry
point for numpy arrays. bf16 tensors are widened exactly (a bf16 value is the top half of a
binary32) before they reach the fp64 code; the MLA cache is passed as raw bf16 bit patterns
so that a million-token cache need not be widened in memory.

Sources are the two pages on Ling-3.1-flash; every C function names the page and section it
follows: "Ling-3.1-flash and the 7:1 hybrid: how much KV cache does a 560B model need at 1M
tokens?" (dev.to) and "Ling-3.1-flash: a 560B hybrid-attention MoE, counted from its
safetensors headers" (ai.thesatyajit.com), section "How KDA and MLA split the work".

Parity status: every function here is pinned by tests under ``tests/test_oracle_*.py``
against closed forms, brute force, special cases and library routines.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lad_oracle.c")
_LIB = os.path.join(_HERE, "liblad_oracle.so")
_lock = threading.Lock()
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_ip = ctypes.POINTER(ctypes.c_int)
_up = ctypes.POINTER(ctypes.c_uint16)
_bp = ctypes.POINTER(ctypes.c_uint8)


def build(force: bool = False) -> str:
    """Compile ``lad_oracle.c`` into ``liblad_oracle.so`` next to it and return the path."""
    stale = (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall",
               "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True, capture_output=True, text=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            lib.lado_kda_recurrent.argtypes = [ctypes.c_int] * 5 + [ctypes.c_double] + [_dp] * 7 + [ctypes.c_int]
            lib.lado_kda_chunked.argtypes = [ctypes.c_int] * 6 + [ctypes.c_double] + [_dp] * 7 + [ctypes.c_int]
            lib.lado_l2norm.argtypes = [ctypes.c_longlong, ctypes.c_int, ctypes.c_double, _dp, _dp]
            lib.lado_short_conv_step.argtypes = [ctypes.c_int] * 3 + [_dp, _dp, _dp, _dp, ctypes.c_int, _dp]
            lib.lado_mla_decode.argtypes = ([ctypes.c_int] * 4 + [ctypes.c_longlong, _dp, _up, _ip, _dp,
                                            ctypes.c_double, _dp, _dp, ctypes.c_int])
            lib.lado_mla_decode_paged.argtypes = ([ctypes.c_int] * 7 + [_dp, _up, _ip, _ip, _dp,
                                                  ctypes.c_double, _dp, _dp, ctypes.c_int])
            lib.lado_rope.argtypes = [ctypes.c_int, ctypes.c_int, _dp, ctypes.POINTER(ctypes.c_longlong),
                                      ctypes.c_double, ctypes.c_int, _dp]
            lib.lado_round_bf16.argtypes = [ctypes.c_int, _dp, _up]
            lib.lado_mla_cache_row.argtypes = [ctypes.c_int] * 3 + [_up, _up, ctypes.POINTER(ctypes.c_longlong),
                                                                    ctypes.c_double, ctypes.c_int, _up]
            lib.lado_gated_rmsnorm.argtypes = [ctypes.c_int, ctypes.c_int, _dp, _dp, _dp, ctypes.c_double, _dp]
            lib.lado_e4m3_decode.argtypes = [ctypes.c_int, _bp, _dp]
            lib.lado_e4m3_encode.argtypes = [ctypes.c_int, _dp, _bp]
            lib.lado_mla_decode_fp8.argtypes = ([ctypes.c_int] * 4 + [ctypes.c_longlong, _dp, _bp, ctypes.c_double,
                                                _ip, _dp, ctypes.c_double, _dp, _dp, ctypes.c_int])
            lib.lado_mla_decode_paged_fp8.argtypes = ([ctypes.c_int] * 7 + [_dp, _bp, ctypes.c_double, _ip, _ip, _dp,
                                                      ctypes.c_double, _dp, _dp, ctypes.c_int])
            lib.lado_mla_cache_row_fp8.argtypes = ([ctypes.c_int] * 3 + [_up, _up, ctypes.POINTER(ctypes.c_longlong),
                                                   ctypes.c_double, ctypes.c_int, ctypes.c_double, _bp])
            lib.lado_num_threads_available.argtypes = []
            for f in (lib.lado_kda_recurrent, lib.lado_kda_chunked, lib.lado_l2norm,
                      lib.lado_short_conv_step, lib.lado_mla_decode, lib.lado_mla_decode_paged, lib.lado_rope,
                      lib.lado_round_bf16, lib.lado_mla_cache_row, lib.lado_gated_rmsnorm,
                      lib.lado_e4m3_decode, lib.lado_e4m3_encode, lib.lado_mla_decode_fp8,
                      lib.lado_mla_decode_paged_fp8, lib.lado_mla_cache_row_fp8,
                      lib.lado_num_threads_available):
                f.restype = ctypes.c_int
            _lib = lib
    return _lib


def max_threads() -> int:
    """Number of OpenMP threads the oracle may use on this host."""
    return int(_load().lado_num_threads_available())


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray, t=_dp):
    return a.ctypes.data_as(t)


def _check(rc: int, name: str) -> None:
    if rc != 0:
        raise RuntimeError(f"oracle {name} failed with status {rc}")


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float64."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def kda_recurrent(q, k, v, alpha, beta, S0, scale: float = 1.0, nthreads: int = 1):
    """Token-by-token KDA gated delta rule.

    q, k, alpha: [B,T,H,dk]; v: [B,T,H,dv]; beta: [B,T,H]; S0: [B,H,dk,dv].
    Returns (o [B,T,H,dv], S_T [B,H,dk,dv]) in float64.
    """
    q, k, v, alpha, beta = map(_f64, (q, k, v, alpha, beta))
    S = _f64(S0).copy()
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    assert k.shape == q.shape and alpha.shape == q.shape and v.shape == (B, T, H, dv)
    assert beta.shape == (B, T, H) and S.shape == (B, H, dk, dv)
    o = np.zeros((B, T, H, dv), dtype=np.float64)
    rc = _load().lado_kda_recurrent(B, T, H, dk, dv, float(scale), _ptr(q), _ptr(k), _ptr(v),
                                    _ptr(alpha), _ptr(beta), _ptr(S), _ptr(o), int(nthreads))
    _check(rc, "kda_recurrent")
    return o, S


def kda_chunked(q, k, v, alpha, beta, S0, chunk: int, scale: float = 1.0, nthreads: int = 1):
    """KDA in chunked WY/UT form; same arguments and results as :func:`kda_recurrent`."""
    q, k, v, alpha, beta = map(_f64, (q, k, v, alpha, beta))
    S = _f64(S0).copy()
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv), dtype=np.float64)
    rc = _load().lado_kda_chunked(B, T, H, dk, dv, int(chunk), float(scale), _ptr(q), _ptr(k),
                                  _ptr(v), _ptr(alpha), _ptr(beta), _ptr(S), _ptr(o), int(nthreads))
    _check(rc, "kda_chunked")
    return o, S


def l2norm(x, eps: float = 1e-6):
    """x / sqrt(sum x^2 + eps) over the last axis."""
    x = _f64(x)
    d = x.shape[-1]
    y = np.empty_like(x)
    _check(_load().lado_l2norm(x.size // d, d, float(eps), _ptr(x), _ptr(y)), "l2norm")
    return y


def short_conv_step(x, tail, w, bias=None, silu: bool = True):
    """One decode step of the width-K causal depthwise convolution.

    x: [B,Cch]; tail: [B,K-1,Cch] (oldest row first); w: [Cch,K]; bias: [Cch] or None.
    Returns (y [B,Cch], new tail [B,K-1,Cch]) in float64.
    """
    x, w = _f64(x), _f64(w)
    tail = _f64(tail).copy()
    B, Cch = x.shape
    K = w.shape[1]
    assert tail.shape == (B, K - 1, Cch) and w.shape == (Cch, K)
    y = np.zeros_like(x)
    bptr = None
    if bias is not None:
        bias = _f64(bias)
        bptr = _ptr(bias)
    rc = _load().lado_short_conv_step(B, Cch, K, _ptr(x), _ptr(tail), _ptr(w), bptr, int(bool(silu)), _ptr(y))
    _check(rc, "short_conv_step")
    return y, tail


def mla_decode(q, cache_bits, seq_lens, gate=None, scale: float = 192 ** -0.5, d_latent: int = 512,
               nthreads: int = 1):
    """Gated latent-attention decode.

    q: [B,H,D] (float, absorbed query, D = d_latent + d_rope); cache_bits: uint16 bf16 bit
    patterns [B,Lmax,D]; seq_lens: [B] ints; gate: [B,H] logits or None.
    Returns (o [B,H,d_latent], lse [B,H]) in float64.
    """
    q = _f64(q)
    cache_bits = np.ascontiguousarray(cache_bits, dtype=np.uint16)
    B, H, D = q.shape
    assert cache_bits.ndim == 3 and cache_bits.shape[0] == B and cache_bits.shape[2] == D
    seq_stride = cache_bits.shape[1] * D
    lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
    assert lens.shape == (B,) and (lens <= cache_bits.shape[1]).all()
    o = np.zeros((B, H, d_latent), dtype=np.float64)
    lse = np.zeros((B, H), dtype=np.float64)
    gptr = None
    if gate is not None:
        gate = _f64(gate)
        gptr = _ptr(gate)
    rc = _load().lado_mla_decode(B, H, d_latent, D - d_latent, seq_stride, _ptr(q),
                                 _ptr(cache_bits, _up), _ptr(lens, _ip), gptr, float(scale),
                                 _ptr(o), _ptr(lse), int(nthreads))
    _check(rc, "mla_decode")
    return o, lse


def mla_decode_paged(q, page_bits, block_table, seq_lens, gate=None, scale: float = 192 ** -0.5,
                     d_latent: int = 512, nthreads: int = 1):
    """mla_decode over a paged cache: page_bits uint16 bf16 bit patterns [num_pages, P, D];
    row t of sequence b is row t % P of page block_table[b, t // P] (block_table int [B, n]).
    Returns (o [B,H,d_latent], lse [B,H]) in float64."""
    q = _f64(q)
    page_bits = np.ascontiguousarray(page_bits, dtype=np.uint16)
    B, H, D = q.shape
    assert page_bits.ndim == 3 and page_bits.shape[2] == D
    num_pages, P = page_bits.shape[0], page_bits.shape[1]
    bt = np.ascontiguousarray(block_table, dtype=np.int32)
    assert bt.ndim == 2 and bt.shape[0] == B
    lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
    assert lens.shape == (B,)
    o = np.zeros((B, H, d_latent), dtype=np.float64)
    lse = np.zeros((B, H), dtype=np.float64)
    gptr = None
    if gate is not None:
        gate = _f64(gate)
        gptr = _ptr(gate)
    rc = _load().lado_mla_decode_paged(B, H, d_latent, D - d_latent, P, num_pages, bt.shape[1], _ptr(q),
                                       _ptr(page_bits, _up), _ptr(bt, _ip), _ptr(lens, _ip), gptr, float(scale),
                                       _ptr(o), _ptr(lse), int(nthreads))
    _check(rc, "mla_decode_paged")
    return o, lse


def e4m3_decode(codes) -> np.ndarray:
    """float64 values of E4M3 codes (uint8, any shape)."""
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(c.shape, dtype=np.float64)
    _check(_load().lado_e4m3_decode(c.size, _ptr(c, _bp), _ptr(out)), "e4m3_decode")
    return out


def e4m3_encode(x) -> np.ndarray:
    """Nearest E4M3 codes of float64 values (ties to even, saturating at +-448, NaN to 0x7F)."""
    x = np.ascontiguousarray(_f64(x))
    out = np.empty(x.shape, dtype=np.uint8)
    _check(_load().lado_e4m3_encode(x.size, _ptr(x), _ptr(out, _bp)), "e4m3_encode")
    return out


def mla_decode_fp8(q, cache_codes, kv_scale: float, seq_lens, gate=None, scale: float = 192 ** -0.5,
                   d_latent: int = 512, nthreads: int = 1):
    """mla_decode over an FP8 cache: cache_codes uint8 E4M3 codes [B,Lmax,D], each element worth
    kv_scale * E4M3(code). Returns (o [B,H,d_latent], lse [B,H]) in float64."""
    q = _f64(q)
    codes = np.ascontiguousarray(cache_codes, dtype=np.uint8)
    B, H, D = q.shape
    assert codes.ndim == 3 and codes.shape[0] == B and codes.shape[2] == D
    lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
    assert lens.shape == (B,) and (lens <= codes.shape[1]).all()
    o = np.zeros((B, H, d_latent), dtype=np.float64)
    lse = np.zeros((B, H), dtype=np.float64)
    gptr = None
    if gate is not None:
        gate = _f64(gate)
        gptr = _ptr(gate)
    rc = _load().lado_mla_decode_fp8(B, H, d_latent, D - d_latent, codes.shape[1] * D, _ptr(q), _ptr(codes, _bp),
                                     float(kv_scale), _ptr(lens, _ip), gptr, float(scale), _ptr(o), _ptr(lse),
                                     int(nthreads))
    _check(rc, "mla_decode_fp8")
    return o, lse


def mla_decode_paged_fp8(q, page_codes, kv_scale: float, block_table, seq_lens, gate=None,
                         scale: float = 192 ** -0.5, d_latent: int = 512, nthreads: int = 1):
    """mla_decode_paged over an FP8 page pool: page_codes uint8 E4M3 codes [num_pages, P, D]."""
    q = _f64(q)
    codes = np.ascontiguousarray(page_codes, dtype=np.uint8)
    B, H, D = q.shape
    assert codes.ndim == 3 and codes.shape[2] == D
    num_pages, P = codes.shape[0], codes.shape[1]
    bt = np.ascontiguousarray(block_table, dtype=np.int32)
    assert bt.ndim == 2 and bt.shape[0] == B
    lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
    assert lens.shape == (B,)
    o = np.zeros((B, H, d_latent), dtype=np.float64)
    lse = np.zeros((B, H), dtype=np.float64)
    gptr = None
    if gate is not None:
        gate = _f64(gate)
        gptr = _ptr(gate)
    rc = _load().lado_mla_decode_paged_fp8(B, H, d_latent, D - d_latent, P, num_pages, bt.shape[1], _ptr(q),
                                           _ptr(codes, _bp), float(kv_scale), _ptr(bt, _ip), _ptr(lens, _ip), gptr,
                                           float(scale), _ptr(o), _ptr(lse), int(nthreads))
    _check(rc, "mla_decode_paged_fp8")
    return o, lse


def rope(x, positions, theta: float = 6.0e6, interleaved: bool = False):
    """Rotary embedding of the last axis of x (even width D) by positions (one per row of the
    leading axes, broadcast over any axes between). Returns float64 of x's shape."""
    x = _f64(x)
    D = x.shape[-1]
    pos = np.asarray(positions, dtype=np.int64)
    lead = x.shape[:-1]
    pos = np.broadcast_to(pos.reshape(pos.shape + (1,) * (len(lead) - pos.ndim)), lead)
    flat = np.ascontiguousarray(x.reshape(-1, D))
    pflat = np.ascontiguousarray(pos.reshape(-1))
    out = np.empty_like(flat)
    rc = _load().lado_rope(flat.shape[0], D, _ptr(flat), pflat.ctypes.data_as(ctypes.POINTER(ctypes.c_longlong)),
                           float(theta), int(bool(interleaved)), _ptr(out))
    _check(rc, "rope")
    return out.reshape(x.shape)


def round_bf16_bits(x) -> np.ndarray:
    """bf16 bit patterns of float64 values, rounded once to nearest, ties to even."""
    x = np.ascontiguousarray(_f64(x))
    out = np.empty(x.shape, dtype=np.uint16)
    _check(_load().lado_round_bf16(x.size, _ptr(x), _ptr(out, _up)), "round_bf16")
    return out


def mla_cache_row_fp8(c_kv_bits, k_pe_bits, positions, kv_scale: float, theta: float = 6.0e6,
                      interleaved: bool = False) -> np.ndarray:
    """New FP8 latent-cache rows (E4M3 codes [n, Dc + Dr]): each element of the row that
    mla_cache_row would round to bf16 is divided by kv_scale in fp32 and rounded to E4M3."""
    c = np.ascontiguousarray(c_kv_bits, dtype=np.uint16)
    k = np.ascontiguousarray(k_pe_bits, dtype=np.uint16)
    n, Dc = c.shape
    Dr = k.shape[1]
    pos = np.ascontiguousarray(positions, dtype=np.int64)
    out = np.empty((n, Dc + Dr), dtype=np.uint8)
    rc = _load().lado_mla_cache_row_fp8(n, Dc, Dr, _ptr(c, _up), _ptr(k, _up),
                                        pos.ctypes.data_as(ctypes.POINTER(ctypes.c_longlong)), float(theta),
                                        int(bool(interleaved)), float(kv_scale), _ptr(out, _bp))
    _check(rc, "mla_cache_row_fp8")
    return out


def mla_cache_row(c_kv_bits, k_pe_bits, positions, theta: float = 6.0e6, interleaved: bool = False) -> np.ndarray:
    """New latent-cache rows (bf16 bits [n, Dc + Dr]): the latent as given, the RoPE key turned
    to its position and rounded to bf16 once. c_kv_bits [n, Dc], k_pe_bits [n, Dr] uint16."""
    c = np.ascontiguousarray(c_kv_bits, dtype=np.uint16)
    k = np.ascontiguousarray(k_pe_bits, dtype=np.uint16)
    n, Dc = c.shape
    Dr = k.shape[1]
    pos = np.ascontiguousarray(positions, dtype=np.int64)
    out = np.empty((n, Dc + Dr), dtype=np.uint16)
    rc = _load().lado_mla_cache_row(n, Dc, Dr, _ptr(c, _up), _ptr(k, _up),
                                    pos.ctypes.data_as(ctypes.POINTER(ctypes.c_longlong)), float(theta),
                                    int(bool(interleaved)), _ptr(out, _up))
    _check(rc, "mla_cache_row")
    return out


def gated_rmsnorm(o, g, w=None, eps: float = 1e-5):
    """KDA output gate: per row of the last axis, o / sqrt(mean(o^2) + eps) * w * sigmoid(g)."""
    o = np.ascontiguousarray(_f64(o))
    g = np.ascontiguousarray(_f64(g))
    assert g.shape == o.shape
    D = o.shape[-1]
    flat_o, flat_g = o.reshape(-1, D), g.reshape(-1, D)
    out = np.empty_like(flat_o)
    wp = None
    if w is not None:
        w = np.ascontiguousarray(_f64(w))
        assert w.shape == (D,)
        wp = _ptr(w)
    rc = _load().lado_gated_rmsnorm(flat_o.shape[0], D, _ptr(flat_o), _ptr(flat_g), wp, float(eps), _ptr(out))
    _check(rc, "gated_rmsnorm")
    return out.reshape(o.shape)
