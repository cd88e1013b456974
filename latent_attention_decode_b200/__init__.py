"""Python binding of the hybrid-attention decode library (``liblad.so``, CUDA for sm_100a).

Each function has the name of a C entry point in ``include/lad.h`` and only marshals arguments:
it checks devices, dtypes and shapes of torch CUDA tensors, allocates outputs or workspace
when the caller passes none, and hands raw pointers plus the current CUDA stream to the
library. All arithmetic runs in the library's kernels; there is no other implementation, and
importing this package fails loudly if ``liblad.so`` is missing (build it with
``python -m latent_attention_decode_b200.build``).

Flags and layouts are documented in ``include/lad.h``.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

__all__ = [
    "kda_conv_update", "kda_decode_step", "kda_conv_decode_step", "kda_conv_decode_step_gated", "kda_decode_multi",
    "kda_prefill_chunked", "kda_prefill_workspace_size",
    "mla_latent_decode", "mla_latent_decode_workspace_size", "mla_latent_decode_paged",
    "mla_latent_decode_paged_rope", "mla_cache_append", "mla_latent_decode_multi",
    "mla_latent_decode_multi_workspace_size", "mla_latent_decode_fp8", "mla_latent_decode_paged_fp8",
    "mla_cache_append_fp8", "mla_latent_decode_noalloc",
    "lad_device_error", "lad_check_bounded_wait", "lad_version",
    "LadError", "LIB_PATH", "FLAG_SILU", "FLAG_L2NORM_QK", "FLAG_OUT_FP32", "FLAG_KEEP_STATE",
    "FLAG_ROPE_INTERLEAVED", "FLAG_OVERLAP_PREV", "MLA_SCALE", "ROPE_THETA",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "liblad.so")

FLAG_SILU = 1 << 0
FLAG_L2NORM_QK = 1 << 1
FLAG_OUT_FP32 = 1 << 2
FLAG_KEEP_STATE = 1 << 3
FLAG_ROPE_INTERLEAVED = 1 << 4
FLAG_OVERLAP_PREV = 1 << 5
ROPE_THETA = 6.0e6
MLA_SCALE = 1.0 / math.sqrt(192.0)

_c_vp = ctypes.c_void_p
_c_int = ctypes.c_int
_c_ll = ctypes.c_longlong
_c_f = ctypes.c_float
_c_u = ctypes.c_uint
_c_sz = ctypes.c_size_t


class LadError(RuntimeError):
    """A library call returned a nonzero status; the message is lad_last_error()."""

    def __init__(self, fn: str, status: int, message: str):
        super().__init__(f"{fn} failed with status {status}: {message}")
        self.status = status


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m latent_attention_decode_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    sig = {
        "lad_last_error": ([], ctypes.c_char_p),
        "lad_version": ([], _c_int),
        "lad_device_error": ([_c_vp, ctypes.POINTER(_c_int)], _c_int),
        "lad_check_bounded_wait": ([ctypes.POINTER(_c_int), ctypes.POINTER(_c_int), _c_vp], _c_int),
        "kda_conv_update": ([_c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_int, _c_int, _c_int, _c_u, _c_vp], _c_int),
        "kda_decode_step": ([_c_vp, _c_vp, _c_vp, _c_ll, _c_vp, _c_vp, _c_vp, _c_vp, _c_int, _c_int, _c_int,
                             _c_int, _c_f, _c_u, _c_vp], _c_int),
        "kda_conv_decode_step": ([_c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_int, _c_int, _c_int,
                                  _c_int, _c_int, _c_f, _c_u, _c_vp], _c_int),
        "kda_conv_decode_step_gated": ([_c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_f, _c_vp,
                                        _c_int, _c_int, _c_int, _c_int, _c_int, _c_f, _c_u, _c_vp], _c_int),
        "kda_decode_multi": ([_c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_int, _c_int, _c_int,
                              _c_int, _c_int, _c_f, _c_u, _c_vp], _c_int),
        "kda_prefill_chunked": ([_c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_int, _c_int, _c_int,
                                 _c_int, _c_int, _c_int, _c_f, _c_u, _c_vp, _c_sz, _c_vp], _c_int),
        "kda_prefill_workspace_size": ([_c_int] * 6, _c_sz),
        "mla_latent_decode": ([_c_vp, _c_vp, _c_ll, _c_vp, _c_vp, _c_vp, _c_vp, _c_int, _c_int, _c_int, _c_int,
                               _c_int, _c_f, _c_u, _c_vp, _c_sz, _c_vp], _c_int),
        "mla_latent_decode_workspace_size": ([_c_int] * 4, _c_sz),
        "mla_latent_decode_paged_rope": ([_c_vp, _c_vp, _c_f, _c_vp, _c_int, _c_int, _c_vp, _c_int, _c_vp, _c_vp,
                                          _c_vp, _c_vp, _c_int, _c_int, _c_int, _c_int, _c_f, _c_u, _c_vp, _c_sz,
                                          _c_vp], _c_int),
        "mla_cache_append": ([_c_vp, _c_vp, _c_vp, _c_vp, _c_ll, _c_int, _c_vp, _c_int, _c_int, _c_int, _c_int,
                              _c_int, _c_int, _c_f, _c_u, _c_vp], _c_int),
        "mla_latent_decode_paged": ([_c_vp, _c_vp, _c_int, _c_int, _c_vp, _c_int, _c_vp, _c_vp, _c_vp, _c_vp,
                                     _c_int, _c_int, _c_int, _c_int, _c_f, _c_u, _c_vp, _c_sz, _c_vp], _c_int),
        "mla_latent_decode_noalloc": ([_c_vp, _c_vp, _c_ll, _c_vp, _c_vp, _c_vp, _c_vp, _c_int, _c_int, _c_int,
                                       _c_int, _c_int, _c_f, _c_u, _c_vp], _c_int),
        "mla_latent_decode_noalloc_max_batch": ([], _c_sz),
        "mla_latent_decode_multi": ([_c_vp, _c_vp, _c_ll, _c_vp, _c_vp, _c_vp, _c_vp, _c_int, _c_int, _c_int, _c_int,
                                     _c_int, _c_int, _c_f, _c_u, _c_vp, _c_sz, _c_vp], _c_int),
        "mla_latent_decode_multi_workspace_size": ([_c_int] * 5, _c_sz),
        "mla_latent_decode_fp8": ([_c_vp, _c_vp, _c_ll, _c_f, _c_vp, _c_vp, _c_vp, _c_vp, _c_int, _c_int, _c_int,
                                   _c_int, _c_int, _c_f, _c_u, _c_vp, _c_sz, _c_vp], _c_int),
        "mla_latent_decode_paged_fp8": ([_c_vp, _c_vp, _c_f, _c_vp, _c_f, _c_int, _c_int, _c_vp, _c_int, _c_vp,
                                         _c_vp, _c_vp, _c_vp, _c_int, _c_int, _c_int, _c_int, _c_f, _c_u, _c_vp,
                                         _c_sz, _c_vp], _c_int),
        "mla_cache_append_fp8": ([_c_vp, _c_vp, _c_vp, _c_vp, _c_ll, _c_int, _c_vp, _c_int, _c_int, _c_int, _c_int,
                                  _c_int, _c_int, _c_f, _c_f, _c_u, _c_vp], _c_int),
    }
    for name, (args, res) in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    return lib


_loaded = None


def _L() -> ctypes.CDLL:
    """The library, loaded on first use (so that building it never needs an old copy)."""
    global _loaded
    if _loaded is None:
        _loaded = _load()
    return _loaded


def __getattr__(name):
    if name == "_lib":
        return _L()
    raise AttributeError(name)


def _check(fn: str, status: int) -> None:
    if status != 0:
        raise LadError(fn, status, _L().lad_last_error().decode(errors="replace"))


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _cuda(t: torch.Tensor, name: str, dtype=None) -> torch.Tensor:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return t


def _contig(t: torch.Tensor, name: str, dtype=None) -> torch.Tensor:
    _cuda(t, name, dtype)
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _ptr(t):
    return None if t is None else t.data_ptr()


def lad_version() -> int:
    return int(_L().lad_version())


def lad_device_error(stream=None) -> int:
    """Synchronises the stream, returns and clears the device error word (0 = no wait gave up)."""
    code = _c_int(0)
    _check("lad_device_error", _L().lad_device_error(_stream(stream), ctypes.byref(code)))
    return int(code.value)


def lad_check_bounded_wait(stream=None) -> tuple[int, list[int]]:
    """Runs the library's bounded-wait check (a barrier wait that can never complete; about 1 s).
    Returns (tag, [warp 0 result, warp 1 result, ms warp 1 waited, abort flag])."""
    tag = _c_int(0)
    res = (_c_int * 4)()
    _check("lad_check_bounded_wait", _L().lad_check_bounded_wait(ctypes.byref(tag), res, _stream(stream)))
    return tag.value, list(res)


def kda_conv_update(x: torch.Tensor, conv_tail: torch.Tensor, w: torch.Tensor, y: torch.Tensor | None = None,
                    bias: torch.Tensor | None = None, silu: bool = True, stream=None) -> torch.Tensor:
    """One step of the width-K causal conv. x [B,Cch], conv_tail [B,K-1,Cch] (updated), w [Cch,K]."""
    bf = torch.bfloat16
    _contig(x, "x", bf), _contig(conv_tail, "conv_tail", bf), _contig(w, "w", bf)
    B, Cch = x.shape
    K = w.shape[1]
    if conv_tail.shape != (B, K - 1, Cch) or w.shape != (Cch, K):
        raise ValueError("kda_conv_update: inconsistent shapes")
    if bias is not None:
        _contig(bias, "bias", bf)
    if y is None:
        y = torch.empty_like(x)
    _contig(y, "y", bf)
    flags = FLAG_SILU if silu else 0
    _check("kda_conv_update", _L().kda_conv_update(x.data_ptr(), conv_tail.data_ptr(), w.data_ptr(), _ptr(bias),
                                                   y.data_ptr(), B, Cch, K, flags, _stream(stream)))
    return y


def _rows(t: torch.Tensor, name: str, B: int, H: int, d: int) -> int:
    """Batch stride (elements) of a [B,H,d] or [B,H*d] bf16 view whose per-sequence block is dense."""
    _cuda(t, name, torch.bfloat16)
    if t.shape == (B, H, d):
        dense = t.stride(2) == 1 and t.stride(1) == d
    elif t.shape == (B, H * d):
        dense = t.stride(1) == 1
    else:
        raise ValueError(f"{name} must be [B,H,{d}] or [B,H*{d}], got {tuple(t.shape)}")
    if not dense:
        raise ValueError(f"{name}: each sequence's H*{d} block must be contiguous")
    return t.stride(0) if B > 1 else H * d


def kda_decode_step(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, alpha: torch.Tensor, beta: torch.Tensor,
                    S: torch.Tensor, o: torch.Tensor | None = None, scale: float = 1.0, l2norm_qk: bool = False,
                    out_fp32: bool = False, overlap_prev: bool = False, stream=None) -> torch.Tensor:
    """One KDA token: S [B,H,128,128] fp32 updated in place; returns o [B,H,128].

    q, k, v may be [B,H,128] or [B,H*128] views sharing one batch stride (for example the
    q, k and v thirds of kda_conv_update's output). overlap_prev: launch as a programmatic
    dependent of the kernel before it on the stream, which must not write S.
    """
    _contig(S, "S", torch.float32)
    B, H, dk, dv = S.shape
    sq, sk, sv = _rows(q, "q", B, H, dk), _rows(k, "k", B, H, dk), _rows(v, "v", B, H, dv)
    if not (sq == sk == sv):
        raise ValueError("q, k and v must share one batch stride")
    _contig(alpha, "alpha", torch.float32), _contig(beta, "beta", torch.float32)
    if alpha.numel() != B * H * dk or beta.numel() != B * H:
        raise ValueError("alpha must be [B,H,dk] and beta [B,H]")
    odt = torch.float32 if out_fp32 else torch.bfloat16
    if o is None:
        o = torch.empty((B, H, dv), device=S.device, dtype=odt)
    _contig(o, "o", odt)
    flags = ((FLAG_L2NORM_QK if l2norm_qk else 0) | (FLAG_OUT_FP32 if out_fp32 else 0)
             | (FLAG_OVERLAP_PREV if overlap_prev else 0))
    _check("kda_decode_step", _L().kda_decode_step(q.data_ptr(), k.data_ptr(), v.data_ptr(), sq, alpha.data_ptr(),
                                                   beta.data_ptr(), S.data_ptr(), o.data_ptr(), B, H, dk, dv,
                                                   float(scale), flags, _stream(stream)))
    return o


def kda_conv_decode_step_gated(x: torch.Tensor, conv_tail: torch.Tensor, conv_w: torch.Tensor, alpha: torch.Tensor,
                               beta: torch.Tensor, S: torch.Tensor, gate: torch.Tensor,
                               norm_w: torch.Tensor | None = None, eps: float = 1e-5, o: torch.Tensor | None = None,
                               conv_bias: torch.Tensor | None = None, silu: bool = True, l2norm_qk: bool = True,
                               scale: float = 1.0, out_fp32: bool = False, overlap_prev: bool = False,
                               stream=None) -> torch.Tensor:
    """kda_conv_decode_step with the output gate (gated RMSNorm) fused: gate bf16 [B,H,128] logits,
    norm_w fp32 [128] (or None). Returns o [B,H,128]. overlap_prev as in kda_conv_decode_step."""
    bf = torch.bfloat16
    _contig(x, "x", bf), _contig(conv_tail, "conv_tail", bf), _contig(conv_w, "conv_w", bf)
    _contig(S, "S", torch.float32), _contig(alpha, "alpha", torch.float32), _contig(beta, "beta", torch.float32)
    _contig(gate, "gate", bf)
    B, H, dk, dv = S.shape
    K = conv_w.shape[1]
    if x.shape != (B, 3 * H * dk) or conv_tail.shape != (B, K - 1, 3 * H * dk) or conv_w.shape != (3 * H * dk, K):
        raise ValueError("kda_conv_decode_step_gated: inconsistent conv shapes")
    if alpha.numel() != B * H * dk or beta.numel() != B * H or gate.shape != (B, H, dv):
        raise ValueError("alpha must be [B,H,dk], beta [B,H], gate [B,H,dv]")
    if norm_w is not None:
        _contig(norm_w, "norm_w", torch.float32)
        if norm_w.shape != (dv,):
            raise ValueError("norm_w must be [dv]")
    if conv_bias is not None:
        _contig(conv_bias, "conv_bias", bf)
    odt = torch.float32 if out_fp32 else bf
    if o is None:
        o = torch.empty((B, H, dv), device=S.device, dtype=odt)
    _contig(o, "o", odt)
    flags = ((FLAG_SILU if silu else 0) | (FLAG_L2NORM_QK if l2norm_qk else 0) | (FLAG_OUT_FP32 if out_fp32 else 0)
             | (FLAG_OVERLAP_PREV if overlap_prev else 0))
    _check("kda_conv_decode_step_gated", _L().kda_conv_decode_step_gated(
        x.data_ptr(), conv_tail.data_ptr(), conv_w.data_ptr(), _ptr(conv_bias), alpha.data_ptr(), beta.data_ptr(),
        S.data_ptr(), gate.data_ptr(), _ptr(norm_w), float(eps), o.data_ptr(), B, H, dk, dv, K, float(scale), flags,
        _stream(stream)))
    return o


def kda_decode_multi(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, alpha: torch.Tensor, beta: torch.Tensor,
                     S: torch.Tensor, o: torch.Tensor | None = None, n_tokens: torch.Tensor | None = None,
                     scale: float = 1.0, l2norm_qk: bool = False, out_fp32: bool = False, keep_state: bool = False,
                     want_output: bool = True, stream=None) -> torch.Tensor | None:
    """T KDA tokens per sequence in one pass over the state: q, k, v [B,T,H,128] bf16, alpha
    [B,T,H,128] fp32, beta [B,T,H] fp32, S [B,H,128,128] fp32 (updated in place unless keep_state).
    n_tokens (int32 [B], optional) limits sequence b to its first n_tokens[b] tokens. Returns
    o [B,T,H,128] (positions past n_tokens[b] untouched), or None when want_output is False."""
    bf = torch.bfloat16
    _contig(S, "S", torch.float32)
    B, H, dk, dv = S.shape
    for t, name in ((q, "q"), (k, "k"), (v, "v")):
        _contig(t, name, bf)
    T = q.shape[1] if q.dim() == 4 else -1
    if q.shape != (B, T, H, dk) or k.shape != q.shape or v.shape != (B, T, H, dv):
        raise ValueError("q, k, v must be [B,T,H,128]")
    _contig(alpha, "alpha", torch.float32), _contig(beta, "beta", torch.float32)
    if alpha.shape != (B, T, H, dk) or beta.shape != (B, T, H):
        raise ValueError("alpha must be [B,T,H,dk] and beta [B,T,H]")
    if n_tokens is not None:
        _contig(n_tokens, "n_tokens", torch.int32)
        if n_tokens.shape != (B,):
            raise ValueError("n_tokens must be [B]")
    odt = torch.float32 if out_fp32 else bf
    if want_output:
        if o is None:
            o = torch.empty((B, T, H, dv), device=S.device, dtype=odt)
        _contig(o, "o", odt)
    else:
        o = None
    flags = ((FLAG_L2NORM_QK if l2norm_qk else 0) | (FLAG_OUT_FP32 if out_fp32 else 0)
             | (FLAG_KEEP_STATE if keep_state else 0))
    _check("kda_decode_multi", _L().kda_decode_multi(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), alpha.data_ptr(), beta.data_ptr(), S.data_ptr(), _ptr(o),
        _ptr(n_tokens), B, T, H, dk, dv, float(scale), flags, _stream(stream)))
    return o


def kda_conv_decode_step(x: torch.Tensor, conv_tail: torch.Tensor, conv_w: torch.Tensor, alpha: torch.Tensor,
                         beta: torch.Tensor, S: torch.Tensor, o: torch.Tensor | None = None,
                         conv_bias: torch.Tensor | None = None, silu: bool = True, l2norm_qk: bool = True,
                         scale: float = 1.0, out_fp32: bool = False, overlap_prev: bool = False,
                         stream=None) -> torch.Tensor:
    """Short conv + KDA step of one layer in one launch. x [B,3*H*128] raw token (q|k|v), conv_tail
    [B,3,3*H*128] and S [B,H,128,128] updated in place; returns o [B,H,128].

    overlap_prev: launch as a programmatic dependent of the kernel before it on the stream. The
    call may start and read S while that kernel runs (all else waits for it), so that kernel must
    not write S: another layer's call, for instance, but not this state's previous step."""
    bf = torch.bfloat16
    _contig(x, "x", bf), _contig(conv_tail, "conv_tail", bf), _contig(conv_w, "conv_w", bf)
    _contig(S, "S", torch.float32), _contig(alpha, "alpha", torch.float32), _contig(beta, "beta", torch.float32)
    B, H, dk, dv = S.shape
    K = conv_w.shape[1]
    if x.shape != (B, 3 * H * dk) or conv_tail.shape != (B, K - 1, 3 * H * dk) or conv_w.shape != (3 * H * dk, K):
        raise ValueError("kda_conv_decode_step: inconsistent conv shapes")
    if alpha.numel() != B * H * dk or beta.numel() != B * H:
        raise ValueError("alpha must be [B,H,dk] and beta [B,H]")
    if conv_bias is not None:
        _contig(conv_bias, "conv_bias", bf)
    odt = torch.float32 if out_fp32 else bf
    if o is None:
        o = torch.empty((B, H, dv), device=S.device, dtype=odt)
    _contig(o, "o", odt)
    flags = ((FLAG_SILU if silu else 0) | (FLAG_L2NORM_QK if l2norm_qk else 0) | (FLAG_OUT_FP32 if out_fp32 else 0)
             | (FLAG_OVERLAP_PREV if overlap_prev else 0))
    _check("kda_conv_decode_step", _L().kda_conv_decode_step(
        x.data_ptr(), conv_tail.data_ptr(), conv_w.data_ptr(), _ptr(conv_bias), alpha.data_ptr(), beta.data_ptr(),
        S.data_ptr(), o.data_ptr(), B, H, dk, dv, K, float(scale), flags, _stream(stream)))
    return o


def kda_prefill_workspace_size(B: int, T: int, H: int, dk: int = 128, dv: int = 128, chunk: int = 64) -> int:
    return int(_L().kda_prefill_workspace_size(B, T, H, dk, dv, chunk))


def kda_prefill_chunked(q, k, v, alpha, beta, S, o=None, chunk: int = 64, scale: float = 1.0,
                        l2norm_qk: bool = False, out_fp32: bool = False, workspace=None, split: bool = True,
                        stream=None):
    """KDA over T tokens in chunks: q,k,alpha [B,T,H,128], v [B,T,H,128], beta [B,T,H]; S in/out.
    split=True runs the two-kernel path with a workspace (allocated here unless given); split=False
    passes no workspace, which selects the single-kernel path."""
    bf = torch.bfloat16
    _contig(q, "q", bf), _contig(k, "k", bf), _contig(v, "v", bf)
    _contig(alpha, "alpha", torch.float32), _contig(beta, "beta", torch.float32), _contig(S, "S", torch.float32)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if k.shape != q.shape or alpha.shape != q.shape or v.shape != (B, T, H, dv) or beta.shape != (B, T, H) \
            or S.shape != (B, H, dk, dv):
        raise ValueError("kda_prefill_chunked: inconsistent shapes")
    odt = torch.float32 if out_fp32 else bf
    if o is None:
        o = torch.empty((B, T, H, dv), device=q.device, dtype=odt)
    _contig(o, "o", odt)
    ws = kda_prefill_workspace_size(B, T, H, dk, dv, chunk)
    if not split:
        workspace = None
    elif workspace is None and ws > 0:
        workspace = torch.empty(ws, device=q.device, dtype=torch.uint8)
    flags = (FLAG_L2NORM_QK if l2norm_qk else 0) | (FLAG_OUT_FP32 if out_fp32 else 0)
    _check("kda_prefill_chunked", _L().kda_prefill_chunked(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), alpha.data_ptr(), beta.data_ptr(), S.data_ptr(), o.data_ptr(),
        B, T, H, dk, dv, chunk, float(scale), flags, _ptr(workspace),
        0 if workspace is None else workspace.numel() * workspace.element_size(), _stream(stream)))
    return o


def mla_latent_decode_workspace_size(B: int, Hq: int = 64, d_latent: int = 512, num_sms: int = 0) -> int:
    return int(_L().mla_latent_decode_workspace_size(B, Hq, d_latent, num_sms))


def mla_latent_decode(q: torch.Tensor, cache: torch.Tensor, seq_lens: torch.Tensor,
                      gate_logits: torch.Tensor | None = None, o: torch.Tensor | None = None,
                      lse: torch.Tensor | None = None, scale: float = MLA_SCALE, d_latent: int = 512,
                      out_fp32: bool = False, workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Gated latent attention: q [B,Hq,576], cache [B,Lmax,576] (rows contiguous), seq_lens int32 [B].

    Returns o [B,Hq,d_latent]; fills lse [B,Hq] when given.
    """
    bf = torch.bfloat16
    _contig(q, "q", bf)
    _cuda(cache, "cache", bf)
    B, Hq, D = q.shape
    if cache.dim() != 3 or cache.shape[0] != B or cache.shape[2] != D or cache.stride(2) != 1 \
            or cache.stride(1) != D:
        raise ValueError("cache must be [B,Lmax,D] with contiguous rows")
    Lmax = cache.shape[1]
    _contig(seq_lens, "seq_lens", torch.int32)
    if seq_lens.shape != (B,):
        raise ValueError("seq_lens must be [B]")
    if gate_logits is not None:
        _contig(gate_logits, "gate_logits", torch.float32)
        if gate_logits.shape != (B, Hq):
            raise ValueError("gate_logits must be [B,Hq]")
    odt = torch.float32 if out_fp32 else bf
    if o is None:
        o = torch.empty((B, Hq, d_latent), device=q.device, dtype=odt)
    _contig(o, "o", odt)
    if lse is not None:
        _contig(lse, "lse", torch.float32)
    ws = mla_latent_decode_workspace_size(B, Hq, d_latent, 0)
    if workspace is None and ws > 0:
        workspace = torch.empty(ws, device=q.device, dtype=torch.uint8)
    flags = FLAG_OUT_FP32 if out_fp32 else 0
    seq_stride = cache.stride(0) if B > 1 else Lmax * D
    _check("mla_latent_decode", _L().mla_latent_decode(
        q.data_ptr(), cache.data_ptr(), seq_stride, seq_lens.data_ptr(), _ptr(gate_logits), o.data_ptr(),
        _ptr(lse), B, Hq, d_latent, D - d_latent, Lmax, float(scale), flags, _ptr(workspace),
        0 if workspace is None else workspace.numel() * workspace.element_size(), _stream(stream)))
    return o


def mla_latent_decode_paged(q: torch.Tensor, kv_pages: torch.Tensor, block_table: torch.Tensor,
                            seq_lens: torch.Tensor, gate_logits: torch.Tensor | None = None,
                            o: torch.Tensor | None = None, lse: torch.Tensor | None = None, scale: float = MLA_SCALE,
                            d_latent: int = 512, out_fp32: bool = False, workspace: torch.Tensor | None = None,
                            stream=None) -> torch.Tensor:
    """Gated latent attention over a paged cache: kv_pages [num_pages, page_size, 576] bf16,
    block_table int32 [B, n] (row t of sequence b is row t % page_size of page
    block_table[b, t // page_size]), seq_lens int32 [B]. Returns o [B,Hq,d_latent]."""
    bf = torch.bfloat16
    _contig(q, "q", bf)
    _contig(kv_pages, "kv_pages", bf)
    B, Hq, D = q.shape
    if kv_pages.dim() != 3 or kv_pages.shape[2] != D:
        raise ValueError("kv_pages must be [num_pages, page_size, D]")
    _contig(block_table, "block_table", torch.int32)
    if block_table.dim() != 2 or block_table.shape[0] != B:
        raise ValueError("block_table must be [B, n]")
    _contig(seq_lens, "seq_lens", torch.int32)
    if seq_lens.shape != (B,):
        raise ValueError("seq_lens must be [B]")
    if gate_logits is not None:
        _contig(gate_logits, "gate_logits", torch.float32)
        if gate_logits.shape != (B, Hq):
            raise ValueError("gate_logits must be [B,Hq]")
    odt = torch.float32 if out_fp32 else bf
    if o is None:
        o = torch.empty((B, Hq, d_latent), device=q.device, dtype=odt)
    _contig(o, "o", odt)
    if lse is not None:
        _contig(lse, "lse", torch.float32)
    ws = mla_latent_decode_workspace_size(B, Hq, d_latent, 0)
    if workspace is None and ws > 0:
        workspace = torch.empty(ws, device=q.device, dtype=torch.uint8)
    _check("mla_latent_decode_paged", _L().mla_latent_decode_paged(
        q.data_ptr(), kv_pages.data_ptr(), kv_pages.shape[0], kv_pages.shape[1], block_table.data_ptr(),
        block_table.shape[1], seq_lens.data_ptr(), _ptr(gate_logits), o.data_ptr(), _ptr(lse), B, Hq, d_latent,
        D - d_latent, float(scale), FLAG_OUT_FP32 if out_fp32 else 0, _ptr(workspace),
        0 if workspace is None else workspace.numel() * workspace.element_size(), _stream(stream)))
    return o


def mla_latent_decode_paged_rope(q: torch.Tensor, positions: torch.Tensor, kv_pages: torch.Tensor,
                                 block_table: torch.Tensor, seq_lens: torch.Tensor,
                                 gate_logits: torch.Tensor | None = None, o: torch.Tensor | None = None,
                                 lse: torch.Tensor | None = None, scale: float = MLA_SCALE,
                                 rope_theta: float = ROPE_THETA, interleaved: bool = False, d_latent: int = 512,
                                 out_fp32: bool = False, workspace: torch.Tensor | None = None,
                                 stream=None) -> torch.Tensor:
    """mla_latent_decode_paged with q's RoPE part (last 64 values per head) turned to positions[b]
    inside the kernel. positions int32 [B]."""
    bf = torch.bfloat16
    _contig(q, "q", bf)
    _contig(kv_pages, "kv_pages", bf)
    B, Hq, D = q.shape
    if kv_pages.dim() != 3 or kv_pages.shape[2] != D:
        raise ValueError("kv_pages must be [num_pages, page_size, D]")
    _contig(block_table, "block_table", torch.int32)
    _contig(seq_lens, "seq_lens", torch.int32)
    _contig(positions, "positions", torch.int32)
    if block_table.dim() != 2 or block_table.shape[0] != B or seq_lens.shape != (B,) or positions.shape != (B,):
        raise ValueError("block_table must be [B, n]; seq_lens and positions [B]")
    if gate_logits is not None:
        _contig(gate_logits, "gate_logits", torch.float32)
    odt = torch.float32 if out_fp32 else bf
    if o is None:
        o = torch.empty((B, Hq, d_latent), device=q.device, dtype=odt)
    _contig(o, "o", odt)
    if lse is not None:
        _contig(lse, "lse", torch.float32)
    ws = mla_latent_decode_workspace_size(B, Hq, d_latent, 0)
    if workspace is None and ws > 0:
        workspace = torch.empty(ws, device=q.device, dtype=torch.uint8)
    flags = (FLAG_OUT_FP32 if out_fp32 else 0) | (FLAG_ROPE_INTERLEAVED if interleaved else 0)
    _check("mla_latent_decode_paged_rope", _L().mla_latent_decode_paged_rope(
        q.data_ptr(), positions.data_ptr(), float(rope_theta), kv_pages.data_ptr(), kv_pages.shape[0],
        kv_pages.shape[1], block_table.data_ptr(), block_table.shape[1], seq_lens.data_ptr(), _ptr(gate_logits),
        o.data_ptr(), _ptr(lse), B, Hq, d_latent, D - d_latent, float(scale), flags, _ptr(workspace),
        0 if workspace is None else workspace.numel() * workspace.element_size(), _stream(stream)))
    return o


def mla_cache_append(c_kv: torch.Tensor, k_pe: torch.Tensor, positions: torch.Tensor, cache: torch.Tensor,
                     block_table: torch.Tensor | None = None, rope_theta: float = ROPE_THETA,
                     interleaved: bool = False, stream=None) -> None:
    """Writes row positions[b] of every sequence: [c_kv[b] ; k_pe[b] turned to positions[b]].
    cache is the contiguous [B, Lmax, 576] cache (block_table None) or a page pool
    [num_pages, page_size, 576] with block_table int32 [B, n]."""
    bf = torch.bfloat16
    _contig(c_kv, "c_kv", bf), _contig(k_pe, "k_pe", bf), _contig(positions, "positions", torch.int32)
    B, Dc = c_kv.shape
    Dr = k_pe.shape[1]
    if k_pe.shape != (B, Dr) or positions.shape != (B,):
        raise ValueError("c_kv [B, 512], k_pe [B, 64], positions [B]")
    flags = FLAG_ROPE_INTERLEAVED if interleaved else 0
    if block_table is None:
        _cuda(cache, "cache", bf)
        if cache.dim() != 3 or cache.shape[0] != B or cache.shape[2] != Dc + Dr or cache.stride(2) != 1 \
                or cache.stride(1) != Dc + Dr:
            raise ValueError("cache must be [B, Lmax, 576] with contiguous rows")
        seq_stride = cache.stride(0) if B > 1 else cache.shape[1] * (Dc + Dr)
        rc = _L().mla_cache_append(c_kv.data_ptr(), k_pe.data_ptr(), positions.data_ptr(), cache.data_ptr(),
                                   seq_stride, cache.shape[1], None, 0, 0, 0, B, Dc, Dr, float(rope_theta), flags,
                                   _stream(stream))
    else:
        _contig(cache, "cache", bf)
        _contig(block_table, "block_table", torch.int32)
        if cache.dim() != 3 or cache.shape[2] != Dc + Dr or block_table.dim() != 2 or block_table.shape[0] != B:
            raise ValueError("cache must be [num_pages, page_size, 576] and block_table [B, n]")
        rc = _L().mla_cache_append(c_kv.data_ptr(), k_pe.data_ptr(), positions.data_ptr(), cache.data_ptr(), 0, 0,
                                   block_table.data_ptr(), block_table.shape[1], cache.shape[0], cache.shape[1], B,
                                   Dc, Dr, float(rope_theta), flags, _stream(stream))
    _check("mla_cache_append", rc)


def _codes(t: torch.Tensor, name: str) -> torch.Tensor:
    """An E4M3 cache as uint8 codes (torch.float8_e4m3fn tensors are viewed, not converted)."""
    if t.dtype == torch.float8_e4m3fn:
        t = t.view(torch.uint8)
    return _cuda(t, name, torch.uint8)


def _mla_common(q, seq_lens, gate_logits, o, lse, d_latent, out_fp32, workspace):
    bf = torch.bfloat16
    _contig(q, "q", bf)
    B, Hq, D = q.shape
    _contig(seq_lens, "seq_lens", torch.int32)
    if seq_lens.shape != (B,):
        raise ValueError("seq_lens must be [B]")
    if gate_logits is not None:
        _contig(gate_logits, "gate_logits", torch.float32)
        if gate_logits.shape != (B, Hq):
            raise ValueError("gate_logits must be [B,Hq]")
    odt = torch.float32 if out_fp32 else bf
    if o is None:
        o = torch.empty((B, Hq, d_latent), device=q.device, dtype=odt)
    _contig(o, "o", odt)
    if lse is not None:
        _contig(lse, "lse", torch.float32)
    ws = mla_latent_decode_workspace_size(B, Hq, d_latent, 0)
    if workspace is None and ws > 0:
        workspace = torch.empty(ws, device=q.device, dtype=torch.uint8)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    return B, Hq, D, o, workspace, ws_bytes


def mla_latent_decode_multi_workspace_size(B: int, T: int, Hq: int = 64, d_latent: int = 512, num_sms: int = 0) -> int:
    return int(_L().mla_latent_decode_multi_workspace_size(B, T, Hq, d_latent, num_sms))


def mla_latent_decode_multi(q: torch.Tensor, cache: torch.Tensor, seq_lens: torch.Tensor,
                            gate_logits: torch.Tensor | None = None, o: torch.Tensor | None = None,
                            lse: torch.Tensor | None = None, scale: float = MLA_SCALE, d_latent: int = 512,
                            out_fp32: bool = False, workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Multi-token step: q [B,T,Hq,576]; the last T of seq_lens[b] cached rows are the tokens' own, token j
    attends rows 0 .. seq_lens[b] - T + j. Returns o [B,T,Hq,d_latent]; fills lse [B,T,Hq] when given."""
    bf = torch.bfloat16
    _contig(q, "q", bf)
    _cuda(cache, "cache", bf)
    B, T, Hq, D = q.shape
    if cache.dim() != 3 or cache.shape[0] != B or cache.shape[2] != D or cache.stride(2) != 1 \
            or cache.stride(1) != D:
        raise ValueError("cache must be [B,Lmax,D] with contiguous rows")
    Lmax = cache.shape[1]
    _contig(seq_lens, "seq_lens", torch.int32)
    if seq_lens.shape != (B,):
        raise ValueError("seq_lens must be [B]")
    if gate_logits is not None:
        _contig(gate_logits, "gate_logits", torch.float32)
        if gate_logits.shape != (B, T, Hq):
            raise ValueError("gate_logits must be [B,T,Hq]")
    odt = torch.float32 if out_fp32 else bf
    if o is None:
        o = torch.empty((B, T, Hq, d_latent), device=q.device, dtype=odt)
    _contig(o, "o", odt)
    if lse is not None:
        _contig(lse, "lse", torch.float32)
    ws = mla_latent_decode_multi_workspace_size(B, T, Hq, d_latent, 0)
    if workspace is None and ws > 0:
        workspace = torch.empty(ws, device=q.device, dtype=torch.uint8)
    seq_stride = cache.stride(0) if B > 1 else Lmax * D
    _check("mla_latent_decode_multi", _L().mla_latent_decode_multi(
        q.data_ptr(), cache.data_ptr(), seq_stride, seq_lens.data_ptr(), _ptr(gate_logits), o.data_ptr(), _ptr(lse),
        B, T, Hq, d_latent, D - d_latent, Lmax, float(scale), FLAG_OUT_FP32 if out_fp32 else 0, _ptr(workspace),
        0 if workspace is None else workspace.numel() * workspace.element_size(), _stream(stream)))
    return o


def mla_latent_decode_fp8(q: torch.Tensor, cache: torch.Tensor, kv_scale: float, seq_lens: torch.Tensor,
                          gate_logits: torch.Tensor | None = None, o: torch.Tensor | None = None,
                          lse: torch.Tensor | None = None, scale: float = MLA_SCALE, d_latent: int = 512,
                          out_fp32: bool = False, workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """mla_latent_decode over an FP8 cache: cache [B,Lmax,576] E4M3 codes (uint8 or
    float8_e4m3fn, rows contiguous), every element worth kv_scale * E4M3(code)."""
    cache = _codes(cache, "cache")
    B, Hq, D, o, workspace, ws_bytes = _mla_common(q, seq_lens, gate_logits, o, lse, d_latent, out_fp32, workspace)
    if cache.dim() != 3 or cache.shape[0] != B or cache.shape[2] != D or cache.stride(2) != 1 \
            or cache.stride(1) != D:
        raise ValueError("cache must be [B,Lmax,D] with contiguous rows")
    Lmax = cache.shape[1]
    seq_stride = cache.stride(0) if B > 1 else Lmax * D
    _check("mla_latent_decode_fp8", _L().mla_latent_decode_fp8(
        q.data_ptr(), cache.data_ptr(), seq_stride, float(kv_scale), seq_lens.data_ptr(), _ptr(gate_logits),
        o.data_ptr(), _ptr(lse), B, Hq, d_latent, D - d_latent, Lmax, float(scale),
        FLAG_OUT_FP32 if out_fp32 else 0, _ptr(workspace), ws_bytes, _stream(stream)))
    return o


def mla_latent_decode_paged_fp8(q: torch.Tensor, kv_pages: torch.Tensor, kv_scale: float, block_table: torch.Tensor,
                                seq_lens: torch.Tensor, positions: torch.Tensor | None = None,
                                gate_logits: torch.Tensor | None = None, o: torch.Tensor | None = None,
                                lse: torch.Tensor | None = None, scale: float = MLA_SCALE,
                                rope_theta: float = ROPE_THETA, interleaved: bool = False, d_latent: int = 512,
                                out_fp32: bool = False, workspace: torch.Tensor | None = None,
                                stream=None) -> torch.Tensor:
    """mla_latent_decode_paged over a pool of FP8 pages [num_pages, page_size, 576] (E4M3 codes);
    with positions (int32 [B]) q's RoPE part is turned in the kernel, as mla_latent_decode_paged_rope."""
    kv_pages = _codes(kv_pages, "kv_pages")
    _contig(kv_pages, "kv_pages")
    B, Hq, D, o, workspace, ws_bytes = _mla_common(q, seq_lens, gate_logits, o, lse, d_latent, out_fp32, workspace)
    if kv_pages.dim() != 3 or kv_pages.shape[2] != D:
        raise ValueError("kv_pages must be [num_pages, page_size, D]")
    _contig(block_table, "block_table", torch.int32)
    if block_table.dim() != 2 or block_table.shape[0] != B:
        raise ValueError("block_table must be [B, n]")
    if positions is not None:
        _contig(positions, "positions", torch.int32)
        if positions.shape != (B,):
            raise ValueError("positions must be [B]")
    flags = (FLAG_OUT_FP32 if out_fp32 else 0) | (FLAG_ROPE_INTERLEAVED if interleaved else 0)
    _check("mla_latent_decode_paged_fp8", _L().mla_latent_decode_paged_fp8(
        q.data_ptr(), _ptr(positions), float(rope_theta), kv_pages.data_ptr(), float(kv_scale), kv_pages.shape[0],
        kv_pages.shape[1], block_table.data_ptr(), block_table.shape[1], seq_lens.data_ptr(), _ptr(gate_logits),
        o.data_ptr(), _ptr(lse), B, Hq, d_latent, D - d_latent, float(scale), flags, _ptr(workspace), ws_bytes,
        _stream(stream)))
    return o


def mla_cache_append_fp8(c_kv: torch.Tensor, k_pe: torch.Tensor, positions: torch.Tensor, cache: torch.Tensor,
                         kv_scale: float, block_table: torch.Tensor | None = None, rope_theta: float = ROPE_THETA,
                         interleaved: bool = False, stream=None) -> None:
    """mla_cache_append into an FP8 cache (E4M3 codes, uint8 or float8_e4m3fn): each element x of
    the new row is stored as the code of x / kv_scale."""
    bf = torch.bfloat16
    cache = _codes(cache, "cache")
    _contig(c_kv, "c_kv", bf), _contig(k_pe, "k_pe", bf), _contig(positions, "positions", torch.int32)
    B, Dc = c_kv.shape
    Dr = k_pe.shape[1]
    if k_pe.shape != (B, Dr) or positions.shape != (B,):
        raise ValueError("c_kv [B, 512], k_pe [B, 64], positions [B]")
    flags = FLAG_ROPE_INTERLEAVED if interleaved else 0
    if block_table is None:
        if cache.dim() != 3 or cache.shape[0] != B or cache.shape[2] != Dc + Dr or cache.stride(2) != 1 \
                or cache.stride(1) != Dc + Dr:
            raise ValueError("cache must be [B, Lmax, 576] with contiguous rows")
        seq_stride = cache.stride(0) if B > 1 else cache.shape[1] * (Dc + Dr)
        rc = _L().mla_cache_append_fp8(c_kv.data_ptr(), k_pe.data_ptr(), positions.data_ptr(), cache.data_ptr(),
                                       seq_stride, cache.shape[1], None, 0, 0, 0, B, Dc, Dr, float(rope_theta),
                                       float(kv_scale), flags, _stream(stream))
    else:
        _contig(cache, "cache")
        _contig(block_table, "block_table", torch.int32)
        if cache.dim() != 3 or cache.shape[2] != Dc + Dr or block_table.dim() != 2 or block_table.shape[0] != B:
            raise ValueError("cache must be [num_pages, page_size, 576] and block_table [B, n]")
        rc = _L().mla_cache_append_fp8(c_kv.data_ptr(), k_pe.data_ptr(), positions.data_ptr(), cache.data_ptr(), 0,
                                       0, block_table.data_ptr(), block_table.shape[1], cache.shape[0],
                                       cache.shape[1], B, Dc, Dr, float(rope_theta), float(kv_scale), flags,
                                       _stream(stream))
    _check("mla_cache_append_fp8", rc)


def mla_latent_decode_noalloc(q: torch.Tensor, cache: torch.Tensor, seq_lens: torch.Tensor,
                              gate_logits: torch.Tensor | None = None, o: torch.Tensor | None = None,
                              lse: torch.Tensor | None = None, scale: float = MLA_SCALE, d_latent: int = 512,
                              out_fp32: bool = False, stream=None) -> torch.Tensor:
    """mla_latent_decode without a workspace, for callers that cannot allocate device memory.

    The library's built-in scratch array limits B to mla_latent_decode_noalloc_max_batch();
    calls that may overlap on the GPU share that array and must be serialised. If ``o`` is
    None it is allocated here by torch; pass ``o`` to keep the whole call allocation-free.
    """
    bf = torch.bfloat16
    _contig(q, "q", bf)
    _cuda(cache, "cache", bf)
    B, Hq, D = q.shape
    if cache.dim() != 3 or cache.shape[0] != B or cache.shape[2] != D or cache.stride(2) != 1 \
            or cache.stride(1) != D:
        raise ValueError("cache must be [B,Lmax,D] with contiguous rows")
    _contig(seq_lens, "seq_lens", torch.int32)
    if gate_logits is not None:
        _contig(gate_logits, "gate_logits", torch.float32)
    odt = torch.float32 if out_fp32 else bf
    if o is None:
        o = torch.empty((B, Hq, d_latent), device=q.device, dtype=odt)
    _contig(o, "o", odt)
    if lse is not None:
        _contig(lse, "lse", torch.float32)
    seq_stride = cache.stride(0) if B > 1 else cache.shape[1] * D
    _check("mla_latent_decode_noalloc", _L().mla_latent_decode_noalloc(
        q.data_ptr(), cache.data_ptr(), seq_stride, seq_lens.data_ptr(), _ptr(gate_logits), o.data_ptr(),
        _ptr(lse), B, Hq, d_latent, D - d_latent, cache.shape[1], float(scale), FLAG_OUT_FP32 if out_fp32 else 0,
        _stream(stream)))
    return o
