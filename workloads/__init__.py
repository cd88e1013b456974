"""Seeded synthetic inputs shaped like the pages' workloads.

This module draws random inputs and nothing else: it holds none of the decode path's
arithmetic, and both the CUDA path (tests, benchmark) and the CPU oracle (tests) take their
inputs from here. Every tensor is drawn from its own torch Philox stream, keyed by a config
seed and the tensor's name, so a tensor does not depend on which others were drawn before it.

Recipes (distributions as the workload descriptions give them):
  q, k        directions uniform on the unit sphere per head (a Gaussian vector divided by its
              length), stored bf16
  v           N(0, 1), bf16
  alpha       per key channel, exp(-softplus(x)) with x ~ N(0, 1), clamped to [0.9, 1) in fp32
              (about 98.6% of the draws land on the 0.9 clamp; ``alpha_mode="uniform"`` draws
              U[0.9, 1) instead so that every channel decays differently)
  beta        sigmoid(x), x ~ N(0, 1), one per head per token, fp32
  KDA state   zero, or N(0, 0.02^2) fp32 for a decode in progress
  conv        new token x ~ N(0, 1) bf16, tails N(0, 1) bf16, taps 0.5 * N(0, 1) bf16
  MLA         latent cache rows N(0, 1) bf16 (512 latent + 64 RoPE), absorbed query N(0, 1)
              bf16, gate logits N(0, 1) fp32, context lengths uniform integers in a range
"""
from __future__ import annotations

import hashlib
import math
from dataclasses import dataclass, field

import numpy as np
import torch

HEADS = 64
HEAD_DIM = 128
D_LATENT = 512
D_ROPE = 64
D_ROW = D_LATENT + D_ROPE
CONV_WIDTH = 4
KDA_CHANNELS = 3 * HEADS * HEAD_DIM  # q, k and v each have 64 x 128 = 8192 channels
MLA_SCALE = 1.0 / math.sqrt(192.0)   # key width 128 (nope) + 64 (rope)
ALPHA_LO = float(np.float32(0.9))
ALPHA_HI = float(np.nextafter(np.float32(1.0), np.float32(0.0)))


def _seed(seed: int, name: str) -> int:
    h = hashlib.sha256(f"{seed}:{name}".encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def _gen(seed: int, name: str, device) -> torch.Generator:
    g = torch.Generator(device=torch.device(device))
    g.manual_seed(_seed(seed, name))
    return g


def normal(shape, seed: int, name: str, device="cpu", std: float = 1.0) -> torch.Tensor:
    """N(0, std^2) float32, drawn in slices of at most 2^28 elements along dim 0 when large."""
    shape = tuple(int(s) for s in shape)
    n = int(np.prod(shape)) if shape else 1
    g = _gen(seed, name, device)
    if n <= (1 << 28) or len(shape) == 0:
        out = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
        return out * std if std != 1.0 else out
    out = torch.empty(shape, device=device, dtype=torch.float32)
    flat = out.view(-1)
    step = 1 << 28
    for i in range(0, n, step):
        m = min(step, n - i)
        flat[i:i + m] = torch.randn((m,), generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        out.mul_(std)
    return out


def normal_bf16(shape, seed: int, name: str, device="cpu", std: float = 1.0) -> torch.Tensor:
    """N(0, std^2) rounded to bf16 (round to nearest even), drawn slice by slice along dim 0."""
    shape = tuple(int(s) for s in shape)
    out = torch.empty(shape, device=device, dtype=torch.bfloat16)
    g = _gen(seed, name, device)
    rows = shape[0]
    per_row = int(np.prod(shape[1:])) if len(shape) > 1 else 1
    step_rows = max(1, (1 << 27) // max(per_row, 1))
    for r in range(0, rows, step_rows):
        m = min(step_rows, rows - r)
        chunk = torch.randn((m,) + shape[1:], generator=g, device=device, dtype=torch.float32)
        if std != 1.0:
            chunk.mul_(std)
        out[r:r + m] = chunk.to(torch.bfloat16)
    return out


E4M3_CODE_STD = 32.0
KV_SCALE_FP8 = 1.0 / E4M3_CODE_STD


def e4m3_codes(shape, seed: int, name: str, device="cpu", std: float = E4M3_CODE_STD) -> torch.Tensor:
    """E4M3 codes (uint8) of N(0, std^2) draws, cast by torch's float8_e4m3fn conversion (round to
    nearest even), drawn slice by slice along dim 0. With std = 32 the draws stay far inside the
    format's +-448; with kv_scale = 1/32 a cache of these codes holds elements distributed like the
    bf16 cache's N(0, 1)."""
    shape = tuple(int(s) for s in shape)
    out = torch.empty(shape, device=device, dtype=torch.uint8)
    g = _gen(seed, name, device)
    rows = shape[0]
    per_row = int(np.prod(shape[1:])) if len(shape) > 1 else 1
    step_rows = max(1, (1 << 27) // max(per_row, 1))
    for r in range(0, rows, step_rows):
        m = min(step_rows, rows - r)
        chunk = torch.randn((m,) + shape[1:], generator=g, device=device, dtype=torch.float32).mul_(std)
        out[r:r + m] = chunk.to(torch.float8_e4m3fn).view(torch.uint8)
    return out


def unit_sphere_bf16(shape, seed: int, name: str, device="cpu") -> torch.Tensor:
    """Directions uniform on the unit sphere over the last axis (Gaussian / its length), bf16."""
    x = normal(shape, seed, name, device).double()
    x = x / x.pow(2).sum(-1, keepdim=True).sqrt()
    return x.to(torch.bfloat16)


def alpha_decay(shape, seed: int, name: str, device="cpu", mode: str = "clamped") -> torch.Tensor:
    """Per-channel decay in [0.9, 1), float32 (see the module docstring for the two modes)."""
    if mode == "uniform":
        g = _gen(seed, name, device)
        u = torch.rand(shape, generator=g, device=device, dtype=torch.float64)
        a = (ALPHA_LO + (1.0 - ALPHA_LO) * u).to(torch.float32)
    elif mode == "clamped":
        x = normal(shape, seed, name, device).double()
        a = torch.exp(-torch.nn.functional.softplus(x)).to(torch.float32)
    else:
        raise ValueError(mode)
    return a.clamp_(ALPHA_LO, ALPHA_HI)


def beta_strength(shape, seed: int, name: str, device="cpu") -> torch.Tensor:
    """Write strength sigmoid(N(0,1)), float32."""
    return torch.sigmoid(normal(shape, seed, name, device).double()).to(torch.float32)


# --------------------------------------------------------------------------------------------
# Workload descriptions
# --------------------------------------------------------------------------------------------

@dataclass(frozen=True)
class KdaScan:
    """KDA over T tokens (recurrent scan or chunked prefill): [B, T, H, 128] inputs."""
    name: str
    B: int
    H: int
    T: int
    chunk: int = 64
    seed: int = 1234
    state_std: float = 0.0
    alpha_mode: str = "clamped"
    dk: int = HEAD_DIM
    dv: int = HEAD_DIM


@dataclass(frozen=True)
class KdaDecode:
    """One decode token through the short conv and the KDA step for B sequences."""
    name: str
    B: int
    H: int = HEADS
    seed: int = 1235
    state_std: float = 0.02
    alpha_mode: str = "clamped"


@dataclass(frozen=True)
class MlaDecode:
    """Gated latent attention for one query token per sequence."""
    name: str
    B: int
    Hq: int = HEADS
    len_lo: int = 8192
    len_hi: int = 131072
    seed: int = 1236
    fixed_len: int | None = None


@dataclass(frozen=True)
class HybridStep:
    """An 8-layer slice: 7 KDA layers and 1 gated MLA layer, one token per sequence."""
    name: str
    B: int
    ctx: int
    kda_layers: int = 7
    seed: int = 1238


CONFIGS = {
    "kda_scan_tiny": KdaScan("kda_scan_tiny", B=1, H=4, T=256, seed=1234),
    "kda_decode_b64": KdaDecode("kda_decode_b64", B=64, seed=1235),
    "mla_decode_b16": MlaDecode("mla_decode_b16", B=16, seed=1236),
    "kda_prefill_32k": KdaScan("kda_prefill_32k", B=1, H=64, T=32768, chunk=64, seed=1237),
    "hybrid_8layer_1m": HybridStep("hybrid_8layer_1m", B=8, ctx=1_000_000, seed=1238),
}


def kda_scan_inputs(cfg: KdaScan, device="cpu") -> dict:
    B, T, H, dk, dv, s = cfg.B, cfg.T, cfg.H, cfg.dk, cfg.dv, cfg.seed
    out = {
        "q": unit_sphere_bf16((B, T, H, dk), s, "q", device),
        "k": unit_sphere_bf16((B, T, H, dk), s, "k", device),
        "v": normal_bf16((B, T, H, dv), s, "v", device),
        "alpha": alpha_decay((B, T, H, dk), s, "alpha", device, cfg.alpha_mode),
        "beta": beta_strength((B, T, H), s, "beta", device),
    }
    if cfg.state_std > 0:
        out["S0"] = normal((B, H, dk, dv), s, "S0", device, std=cfg.state_std)
    else:
        out["S0"] = torch.zeros((B, H, dk, dv), device=device, dtype=torch.float32)
    return out


def conv_inputs(B: int, seed: int, device="cpu", channels: int = KDA_CHANNELS,
                width: int = CONV_WIDTH, tag: str = "") -> dict:
    """Raw new token x (q|k|v channels), the kept tails and the depthwise taps."""
    return {
        "x": normal_bf16((B, channels), seed, tag + "conv_x", device),
        "tail": normal_bf16((B, width - 1, channels), seed, tag + "conv_tail", device),
        "w": normal_bf16((channels, width), seed, tag + "conv_w", device, std=0.5),
    }


def kda_decode_inputs(cfg: KdaDecode, device="cpu", tag: str = "") -> dict:
    """Inputs of one KDA decode layer: conv token and tails, decay, strength and state.

    The new token x enters the short convolution; its q and k thirds are drawn on the unit
    sphere per head, its v third N(0, 1), matching the scan recipe.
    """
    B, H, s = cfg.B, cfg.H, cfg.seed
    d = HEAD_DIM
    q = unit_sphere_bf16((B, H, d), s, tag + "q", device)
    k = unit_sphere_bf16((B, H, d), s, tag + "k", device)
    v = normal_bf16((B, H, d), s, tag + "v", device)
    conv = conv_inputs(B, s, device, channels=3 * H * d, tag=tag)
    conv["x"] = torch.cat([q.reshape(B, -1), k.reshape(B, -1), v.reshape(B, -1)], dim=1).contiguous()
    return {
        **conv,
        "alpha": alpha_decay((B, H, d), s, tag + "alpha", device, cfg.alpha_mode),
        "beta": beta_strength((B, H), s, tag + "beta", device),
        "S": (normal((B, H, d, d), s, tag + "S", device, std=cfg.state_std) if cfg.state_std > 0
              else torch.zeros((B, H, d, d), device=device, dtype=torch.float32)),
    }


def mla_seq_lens(cfg: MlaDecode) -> torch.Tensor:
    if cfg.fixed_len is not None:
        return torch.full((cfg.B,), cfg.fixed_len, dtype=torch.int32)
    g = torch.Generator()
    g.manual_seed(_seed(cfg.seed, "seq_lens"))
    return torch.randint(cfg.len_lo, cfg.len_hi + 1, (cfg.B,), generator=g, dtype=torch.int64).to(torch.int32)


def mla_inputs(cfg: MlaDecode, device="cpu", lmax: int | None = None) -> dict:
    lens = mla_seq_lens(cfg)
    L = int(lens.max().item()) if lmax is None else int(lmax)
    s = cfg.seed
    return {
        "q": normal_bf16((cfg.B, cfg.Hq, D_ROW), s, "mla_q", device),
        "cache": normal_bf16((cfg.B, L, D_ROW), s, "mla_cache", device),
        "seq_lens": lens.to(device),
        "gate": normal((cfg.B, cfg.Hq), s, "mla_gate", device),
    }


def mla_fp8_cache(cfg: MlaDecode, device="cpu", lmax: int | None = None) -> torch.Tensor:
    """The FP8 latent cache of an MLA workload: E4M3 codes [B, Lmax, 576] (kv_scale KV_SCALE_FP8)."""
    L = int(mla_seq_lens(cfg).max().item()) if lmax is None else int(lmax)
    return e4m3_codes((cfg.B, L, D_ROW), cfg.seed, "mla_cache_fp8", device)


def paginate(cache: torch.Tensor, seq_lens: torch.Tensor, page_size: int, seed: int, spare_pages: int = 0):
    """Moves a contiguous latent cache [B, Lmax, D] into a pool of pages of `page_size` rows placed
    in a seeded random order, the way a serving engine's allocator scatters them. Rows of a page
    past its sequence's length, and spare pages, hold NaN (for a uint8 cache of E4M3 codes, the
    NaN code 0x7F). Returns (pool [P, page_size, D], block_table int32 [B, max pages], on the
    cache's device); unused table entries are -1."""
    B, _, D = cache.shape
    fill = 0x7F if cache.dtype == torch.uint8 else float("nan")
    lens = [int(x) for x in seq_lens.tolist()]
    per_seq = [(n + page_size - 1) // page_size for n in lens]
    n_pages = sum(per_seq) + spare_pages
    perm = np.random.default_rng(_seed(seed, "pages")).permutation(n_pages)
    pool = torch.full((n_pages, page_size, D), fill, dtype=cache.dtype, device=cache.device)
    table = torch.full((B, max(max(per_seq, default=0), 1)), -1, dtype=torch.int32)
    k = 0
    for b in range(B):
        n = per_seq[b]
        if n == 0:
            continue
        pages = torch.from_numpy(perm[k:k + n].astype(np.int64))
        k += n
        table[b, :n] = pages.to(torch.int32)
        rows = cache[b, :lens[b]]
        full = lens[b] // page_size
        dev_pages = pages.to(cache.device)
        if full:
            pool[dev_pages[:full]] = rows[:full * page_size].reshape(full, page_size, D)
        if lens[b] > full * page_size:
            pool[dev_pages[full], :lens[b] - full * page_size] = rows[full * page_size:]
    return pool, table.to(cache.device)


def to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact widening of a (bf16 or fp32) tensor to a float64 numpy array."""
    return t.detach().to("cpu").to(torch.float64).numpy()


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """Raw bf16 bit patterns of a bf16 tensor as uint16 numpy (no copy of values' meaning)."""
    assert t.dtype == torch.bfloat16
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)
