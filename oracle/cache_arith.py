"""Closed-form memory accounting of the hybrid-attention caches.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Follows "Ling-3.1-flash and the 7:1 hybrid: how much KV cache does a 560B model need at 1M
tokens?" (dev.to), sections "How big is the cache per token, exactly?" (latent row = 512 + 64
elements per token per MLA layer, bf16; one 128 x 128 fp32 state per head per KDA layer) and
"What does that mean for serving?" (cache budget and concurrency), and "Ling-3.1-flash: a 560B
hybrid-attention MoE, counted from its safetensors headers", section "Does 292 GiB fit on four
Hopper GPUs?" (MTP layer adds one more latent row; convolution tails).
"""
from __future__ import annotations

from dataclasses import dataclass


@dataclass(frozen=True)
class HybridShape:
    layers: int = 72          # 63 KDA + 9 gated MLA, one MLA layer every 8th layer
    mla_layers: int = 9
    kda_layers: int = 63
    heads: int = 64
    head_dim: int = 128       # d_k = d_v of the KDA state
    kv_lora_rank: int = 512   # latent part of an MLA cache row
    qk_rope_head_dim: int = 64
    conv_width: int = 4
    cache_bytes: int = 2      # bf16 latent cache
    state_bytes: int = 4      # fp32 KDA state
    conv_bytes: int = 2       # bf16 convolution tail
    key_width: int = 192      # per-head key of the expanded (plain MHA) form: 128 nope + 64 rope
    value_width: int = 128


def mla_layer_index(layer: int) -> bool:
    """Layer ``layer`` (0-based) is gated MLA when (layer + 1) % 8 == 0, else KDA."""
    return (layer + 1) % 8 == 0


def latent_row_elems(s: HybridShape = HybridShape()) -> int:
    return s.kv_lora_rank + s.qk_rope_head_dim


def per_token_bytes_hybrid(s: HybridShape = HybridShape(), with_mtp: bool = False) -> int:
    layers = s.mla_layers + (1 if with_mtp else 0)
    return layers * latent_row_elems(s) * s.cache_bytes


def per_token_bytes_all_mla(s: HybridShape = HybridShape()) -> int:
    return s.layers * latent_row_elems(s) * s.cache_bytes


def kda_state_bytes(s: HybridShape = HybridShape()) -> int:
    """Constant per-sequence KDA state over all KDA layers."""
    return s.kda_layers * s.heads * s.head_dim * s.head_dim * s.state_bytes


def conv_tail_bytes(s: HybridShape = HybridShape()) -> int:
    """Per-sequence convolution tails: K-1 past inputs of q, k and v per KDA layer."""
    return s.kda_layers * 3 * s.heads * s.head_dim * (s.conv_width - 1) * s.conv_bytes


def cache_gb(ctx: int, hybrid: bool = True, s: HybridShape = HybridShape()) -> float:
    if hybrid:
        return (per_token_bytes_hybrid(s) * ctx + kda_state_bytes(s)) / 1e9
    return per_token_bytes_all_mla(s) * ctx / 1e9


def mha_bytes_per_token(s: HybridShape = HybridShape()) -> int:
    """Hypothetical plain MHA: full keys and values in every layer."""
    return s.layers * s.heads * (s.key_width + s.value_width) * s.cache_bytes


def break_even_tokens(s: HybridShape = HybridShape()) -> float:
    """Context length whose MLA cache equals the constant KDA state."""
    return kda_state_bytes(s) / per_token_bytes_hybrid(s)


def concurrency(budget_bytes: float, ctx: int, hybrid: bool = True, s: HybridShape = HybridShape()) -> int:
    """Whole sequences of length ``ctx`` that fit in a cache budget."""
    per_seq = cache_gb(ctx, hybrid, s) * 1e9
    return int(budget_bytes // per_seq)


def serving_budget_bytes(gpus: int = 8, gpu_gb: float = 141.0, utilization: float = 0.85,
                         weights_gb: float = 573.8) -> float:
    return (gpus * gpu_gb * utilization - weights_gb) * 1e9


def mla_cache_bytes(batch: int, ctx: int, s: HybridShape = HybridShape()) -> int:
    """Bytes of one MLA layer's latent cache for ``batch`` sequences of ``ctx`` tokens."""
    return batch * ctx * latent_row_elems(s) * s.cache_bytes
