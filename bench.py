#!/usr/bin/env python
"""Benchmark of the hybrid-attention decode path on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl lad|reference]

A step is one pass of the workload's hot path over one batch of synthetic input:
  hybrid_8layer_1m (default)  8-layer slice of the 7:1 hybrid, one decode token for 8 sequences:
                              7 x (kda_conv_update + kda_decode_step) + 1 x mla_latent_decode over
                              1,000,000 cached tokens per sequence
  kda_decode_b64              one KDA layer: kda_conv_update + kda_decode_step, 64 sequences x 64 heads
  mla_decode_b16              one gated MLA layer, 16 sequences, contexts uniform in [8192, 131072]
  mla_decode_b16_paged        the same layer with the cache in 64-row pages of a shuffled pool
  mla_decode_b16_paged_rope   the paged layer with RoPE in the kernels: append the new rows, then attend
  mla_mtp_b16                 mla_decode_b16 with 4 query tokens per sequence (mla_latent_decode_multi)
  mla_decode_b16_fp8          mla_decode_b16 over an FP8 (E4M3) cache, one fp32 scale (mla_latent_decode_fp8)
  mla_decode_b16_paged_rope_fp8  the engine step of mla_decode_b16_paged_rope over FP8 pages
  kda_decode_b64_gated        the same layer with the output gate fused (kda_conv_decode_step_gated)
  kda_mtp_b64                 kda_decode_multi: 64 sequences x 64 heads, 4 tokens per state pass
  kda_prefill_32k             kda_prefill_chunked, 1 x 32768 tokens x 64 heads, chunk 64

Multi-GPU (torchrun, one process per GPU): the path shards by sequence with no exchange, so each
rank runs the same per-GPU workload on its own sequences ("weak" scaling); the step time is the
max over ranks and `value` counts the tokens of all ranks.

`--impl reference` times the fp64 CPU oracle (the only other implementation of the path) on the
host cores, on a bounded sample of the same workload, and prints the same line with
"impl": "reference".
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads as wl  # noqa: E402

METRIC = "decode tokens/s and achieved HBM GB/s (% of B200 roofline) per layer type"
DEFAULT_WORKLOAD = "hybrid_8layer_1m"
H, D = wl.HEADS, wl.HEAD_DIM


# ---------------------------------------------------------------------------------------------
# host-side plumbing shared with the multi-process tests
# ---------------------------------------------------------------------------------------------

def dist_env() -> tuple[int, int, int]:
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def shard_sequences(global_batch: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous range [lo, hi) of the global batch that `rank` owns (sizes differ by <= 1)."""
    base, rem = divmod(global_batch, world)
    lo = rank * base + min(rank, rem)
    return lo, lo + base + (1 if rank < rem else 0)


def max_over_ranks(x: float, device=None) -> float:
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, device=None) -> float:
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def barrier(device_index=None) -> None:
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device_index is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device_index])
        else:
            dist.barrier()


def physical_gpu_index(local: int) -> int:
    """nvidia-smi index of this process's GPU (CUDA_VISIBLE_DEVICES maps local ordinals)."""
    vis = [v.strip() for v in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if v.strip()]
    if local < len(vis) and vis[local].isdigit():
        return int(vis[local])
    return local


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def kernel_traffic(kernel: str, units: float | None) -> dict | None:
    """DRAM bytes of one launch of `kernel` from the ncu capture recorded in profiles/traffic.json,
    scaled by units (cached rows, heads, token-heads) to this launch; None when there is no capture
    or the kernel's source has changed since it was taken."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if units is None or not os.path.exists(p):
        return None
    with open(p) as f:
        e = json.load(f)["kernels"].get(kernel)
    if not e:
        return None
    with open(os.path.join(ROOT, e["source"]), "rb") as f:
        if hashlib.sha256(f.read()).hexdigest() != e["sha256"]:
            return None
    scale = units / e["units"]
    out = {"bytes": int(round((e["read"] + e["write"]) * scale)), "scaled_from": e["capture"],
           "scale": round(scale, 6), "profile": e["profile"]}
    if "tensor_pipe_active_pct" in e:
        out["tensor_pipe_active_pct"] = e["tensor_pipe_active_pct"]
    return out


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None
        self.lines: list[str] = []
        self._t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", str(self.gpu_index)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self._t = threading.Thread(target=self._read, daemon=True)
        self._t.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self._t:
            self._t.join(timeout=5)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------------------------
# workloads: each builds its resident device state and returns a Step
# ---------------------------------------------------------------------------------------------

class Step:
    """One workload on one GPU.

    run(): enqueue one step on the current stream (inputs already resident).
    run_e2e(): the same step with this step's inputs copied in from pinned host memory and the
    step's outputs read back to pinned host memory, all on the current stream.
    """

    name = ""
    tokens_per_step = 0          # decode tokens (or prefill tokens) one step produces on this GPU
    launches_per_step = 0        # library kernels one step launches
    dominant = ""                # name of the roofline kernel

    def dominant_units(self):
        """Units of the dominant kernel's work per launch, in the unit profiles/traffic.json uses."""
        return None
    dominant_unit = "GB/s"
    dominant_bound = "hbm"
    config: dict = {}

    def run(self, timer=None):
        raise NotImplementedError

    def run_e2e(self):
        raise NotImplementedError

    def algorithmic_bytes(self) -> dict:
        """Algorithmic bytes per launch of each kernel kind, and per step."""
        raise NotImplementedError


class _KdaLayer:
    """State and per-token inputs of one KDA decode layer (conv + gated delta rule).

    fused=True runs kda_conv_decode_step (one launch); fused=False runs kda_conv_update and
    kda_decode_step on the conv output (two launches)."""

    fused = True
    # launch the step as a programmatic dependent of the kernel before it (LAD_FLAG_OVERLAP_PREV):
    # only where that kernel never writes this layer's state, i.e. between different layers
    overlap = False

    def __init__(self, lad, B, seed, dev, tag=""):
        cfg = wl.KdaDecode(f"kda{tag}", B=B, seed=seed)
        inp = wl.kda_decode_inputs(cfg, dev, tag=tag)
        self.lad, self.B = lad, B
        self.x, self.tail, self.w = inp["x"], inp["tail"], inp["w"]
        self.alpha, self.beta, self.S = inp["alpha"], inp["beta"], inp["S"]
        self.y = torch.empty_like(self.x)
        self.o = torch.empty((B, H, D), device=dev, dtype=torch.bfloat16)
        # pinned host copies of the per-token inputs and outputs (for the end-to-end timing)
        self.h_x = self.x.cpu().pin_memory()
        self.h_alpha = self.alpha.cpu().pin_memory()
        self.h_beta = self.beta.cpu().pin_memory()
        self.h_o = torch.empty(self.o.shape, dtype=self.o.dtype).pin_memory()

    def run(self, timer=None):
        lad, hd = self.lad, H * D
        if self.fused:
            if timer:
                timer.begin("kda_conv_decode_step")
            lad.kda_conv_decode_step(self.x, self.tail, self.w, self.alpha, self.beta, self.S, o=self.o,
                                     overlap_prev=self.overlap)
            if timer:
                timer.end("kda_conv_decode_step")
            return
        lad.kda_conv_update(self.x, self.tail, self.w, y=self.y, silu=True)
        if timer:
            timer.begin("kda_decode_step")
        lad.kda_decode_step(self.y[:, :hd], self.y[:, hd:2 * hd], self.y[:, 2 * hd:], self.alpha, self.beta,
                            self.S, o=self.o, l2norm_qk=True, overlap_prev=self.overlap)
        if timer:
            timer.end("kda_decode_step")

    def h2d(self):
        self.x.copy_(self.h_x, non_blocking=True)
        self.alpha.copy_(self.h_alpha, non_blocking=True)
        self.beta.copy_(self.h_beta, non_blocking=True)

    def d2h(self):
        self.h_o.copy_(self.o, non_blocking=True)

    def h2d_bytes(self):
        return sum(t.numel() * t.element_size() for t in (self.h_x, self.h_alpha, self.h_beta))

    def d2h_bytes(self):
        return self.h_o.numel() * self.h_o.element_size()

    @staticmethod
    def bytes_conv(B):
        C = 3 * H * D
        # x, tail read, tail written, y per sequence (bf16); taps once per launch
        return B * C * 2 * (1 + 3 + 3 + 1) + C * 4 * 2

    @staticmethod
    def bytes_fused(B):
        # state read + write, raw token, tails read + written, alpha, beta, o per (b, h); taps once
        C = 3 * H * D
        return B * H * (2 * D * D * 4 + D * 4 + 4 + D * 2) + B * C * 2 * (1 + 3 + 3) + C * 4 * 2

    @staticmethod
    def bytes_decode(B):
        # per (b, h): state read + write (fp32 128x128), q,k,v (bf16), alpha (fp32), beta, o (bf16)
        return B * H * (2 * D * D * 4 + 3 * D * 2 + D * 4 + 4 + D * 2)


class KdaDecodeStep(Step):
    name = "kda_decode_b64"

    def __init__(self, lad, dev, rank, B=64):
        self.layer = _KdaLayer(lad, B, 1235 + 1000 * rank, dev)
        self.tokens_per_step = B
        self.launches_per_step = 1 if _KdaLayer.fused else 2
        self.dominant = "kda_conv_decode_step" if _KdaLayer.fused else "kda_decode_step"
        self.config = {"workload": self.name, "batch_per_gpu": B, "heads": H, "head_dim": D,
                       "kda_path": "fused conv+step" if _KdaLayer.fused else "conv, then step",
                       "state": "fp32 128x128 per head", "conv": "width 4 over 3x8192 bf16 channels",
                       "l2": "inputs larger than L2 (268 MB of state per step)"}

    def run(self, timer=None):
        self.layer.run(timer)

    def run_e2e(self):
        self.layer.h2d()
        self.layer.run()
        self.layer.d2h()

    def e2e_bytes(self):
        return self.layer.h2d_bytes(), self.layer.d2h_bytes()

    def dominant_units(self):
        return self.layer.B * H

    def algorithmic_bytes(self):
        B = self.layer.B
        return {"kda_decode_step": _KdaLayer.bytes_decode(B), "kda_conv_update": _KdaLayer.bytes_conv(B),
                "kda_conv_decode_step": _KdaLayer.bytes_fused(B),
                "step": (_KdaLayer.bytes_fused(B) if _KdaLayer.fused
                         else _KdaLayer.bytes_decode(B) + _KdaLayer.bytes_conv(B))}


class KdaGatedStep(KdaDecodeStep):
    """The 64 x 64-head KDA layer with the output gate (gated RMSNorm) fused into the step:
    kda_conv_decode_step_gated."""
    name = "kda_decode_b64_gated"

    def __init__(self, lad, dev, rank, B=64):
        super().__init__(lad, dev, rank, B)
        L = self.layer
        self.gate = wl.normal_bf16((B, H, D), 1235 + 1000 * rank, "kda_gate", dev, std=2.0)
        self.norm_w = torch.ones(D, device=dev, dtype=torch.float32)
        self.h_gate = self.gate.cpu().pin_memory()
        self.dominant = "kda_conv_decode_step_gated"
        self.launches_per_step = 1
        self.config = dict(self.config, workload=self.name, kda_path="fused conv+step+output gate")

    def run(self, timer=None):
        L = self.layer
        if timer:
            timer.begin("kda_conv_decode_step_gated")
        L.lad.kda_conv_decode_step_gated(L.x, L.tail, L.w, L.alpha, L.beta, L.S, self.gate, self.norm_w, o=L.o)
        if timer:
            timer.end("kda_conv_decode_step_gated")

    def run_e2e(self):
        self.layer.h2d()
        self.gate.copy_(self.h_gate, non_blocking=True)
        self.run()
        self.layer.d2h()

    def e2e_bytes(self):
        return self.layer.h2d_bytes() + self.h_gate.numel() * 2, self.layer.d2h_bytes()

    def dominant_units(self):
        return self.layer.B * H

    def algorithmic_bytes(self):
        b = _KdaLayer.bytes_fused(self.layer.B) + self.layer.B * H * D * 2 + D * 4
        return {"kda_conv_decode_step_gated": b, "step": b}


class KdaMultiStep(Step):
    """One KDA layer's multi-token pass: 64 sequences x 64 heads, 4 tokens per sequence (one
    token plus three drafts, the verify step of multi-token prediction) through
    kda_decode_multi, the state read once and written once."""
    name = "kda_mtp_b64"

    def __init__(self, lad, dev, rank, B=64, T=4):
        cfg = wl.KdaScan("mtp", B=B, H=H, T=T, seed=1240 + 1000 * rank, state_std=0.02)
        inp = wl.kda_scan_inputs(cfg, dev)
        self.lad, self.B, self.T = lad, B, T
        self.q, self.k, self.v = inp["q"], inp["k"], inp["v"]
        self.alpha, self.beta, self.S = inp["alpha"], inp["beta"], inp["S0"]
        self.o = torch.empty((B, T, H, D), device=dev, dtype=torch.bfloat16)
        self.h_in = [t.cpu().pin_memory() for t in (self.q, self.k, self.v, self.alpha, self.beta)]
        self.h_o = torch.empty(self.o.shape, dtype=self.o.dtype).pin_memory()
        self.tokens_per_step = B * T
        self.launches_per_step = 1
        self.dominant = "kda_decode_multi"
        self.config = {"workload": self.name, "batch_per_gpu": B, "tokens_per_pass": T, "heads": H,
                       "head_dim": D, "state": "fp32 128x128 per head, read and written once per pass",
                       "l2": "inputs larger than L2 (268 MB of state per step)"}

    def run(self, timer=None):
        if timer:
            timer.begin("kda_decode_multi")
        self.lad.kda_decode_multi(self.q, self.k, self.v, self.alpha, self.beta, self.S, o=self.o)
        if timer:
            timer.end("kda_decode_multi")

    def run_e2e(self):
        for d, h in zip((self.q, self.k, self.v, self.alpha, self.beta), self.h_in):
            d.copy_(h, non_blocking=True)
        self.run()
        self.h_o.copy_(self.o, non_blocking=True)

    def e2e_bytes(self):
        return sum(t.numel() * t.element_size() for t in self.h_in), self.h_o.numel() * 2

    def dominant_units(self):
        return self.B * H if self.T == 4 else None

    def algorithmic_bytes(self):
        # per (b, h): state read + write; per token q, k, v (bf16), alpha (fp32), beta, o (bf16)
        b = self.B * H * (2 * D * D * 4 + self.T * (3 * D * 2 + D * 4 + 4 + D * 2))
        return {"kda_decode_multi": b, "step": b}


class MlaDecodeStep(Step):
    name = "mla_decode_b16"

    def __init__(self, lad, dev, rank, cfg: wl.MlaDecode | None = None):
        cfg = cfg or wl.MlaDecode("mla", B=16, seed=1236 + 1000 * rank)
        self.lad, self.cfg = lad, cfg
        inp = wl.mla_inputs(cfg, dev)
        self.q, self.cache, self.lens, self.gate = inp["q"], inp["cache"], inp["seq_lens"], inp["gate"]
        self.total_len = int(self.lens.sum().item())
        self.o = torch.empty((cfg.B, cfg.Hq, wl.D_LATENT), device=dev, dtype=torch.bfloat16)
        self.ws = torch.empty(lad.mla_latent_decode_workspace_size(cfg.B, cfg.Hq, wl.D_LATENT, 0), device=dev,
                              dtype=torch.uint8)
        self.h_q = self.q.cpu().pin_memory()
        self.h_gate = self.gate.cpu().pin_memory()
        self.h_o = torch.empty(self.o.shape, dtype=self.o.dtype).pin_memory()
        self.tokens_per_step = cfg.B
        self.launches_per_step = 2
        self.dominant = "mla_latent_decode"
        self.config = {"workload": self.name, "batch_per_gpu": cfg.B, "q_heads": cfg.Hq,
                       "cache_row": "512 latent + 64 rope, bf16",
                       "context": (f"{cfg.fixed_len} per sequence" if cfg.fixed_len else
                                   f"uniform [{cfg.len_lo}, {cfg.len_hi}], total {self.total_len}"),
                       "l2": "inputs larger than L2 (latent cache)"}

    def run(self, timer=None):
        if timer:
            timer.begin("mla_latent_decode")
        self.lad.mla_latent_decode(self.q, self.cache, self.lens, self.gate, o=self.o, workspace=self.ws)
        if timer:
            timer.end("mla_latent_decode")

    def h2d(self):
        self.q.copy_(self.h_q, non_blocking=True)
        self.gate.copy_(self.h_gate, non_blocking=True)

    def d2h(self):
        self.h_o.copy_(self.o, non_blocking=True)

    def run_e2e(self):
        self.h2d()
        self.run()
        self.d2h()

    def e2e_bytes(self):
        hb = self.h_q.numel() * 2 + self.h_gate.numel() * 4
        return hb, self.h_o.numel() * 2

    def mla_bytes(self):
        B, Hq = self.cfg.B, self.cfg.Hq
        return self.total_len * wl.D_ROW * 2 + B * Hq * (wl.D_ROW * 2 + 4 + wl.D_LATENT * 2) + B * 4

    def mla_flops(self):
        return 2 * self.cfg.Hq * (wl.D_ROW + wl.D_LATENT) * self.total_len

    def dominant_units(self):
        return self.total_len

    def algorithmic_bytes(self):
        b = self.mla_bytes()
        return {"mla_latent_decode": b, "step": b}


class MlaPagedStep(MlaDecodeStep):
    """The 16-sequence latent-attention workload with the cache in 64-row pages scattered through
    a pool (seeded order), through mla_latent_decode_paged."""
    name = "mla_decode_b16_paged"
    page_size = 64

    def __init__(self, lad, dev, rank, cfg: wl.MlaDecode | None = None):
        super().__init__(lad, dev, rank, cfg)
        self.pool, self.block_table = wl.paginate(self.cache, self.lens, self.page_size, self.cfg.seed)
        del self.cache
        torch.cuda.empty_cache()
        self.dominant = "mla_latent_decode_paged"
        self.config = dict(self.config, workload=self.name,
                           paging=f"{self.page_size}-row pages, {self.pool.shape[0]} in a shuffled pool")

    def run(self, timer=None):
        if timer:
            timer.begin("mla_latent_decode_paged")
        self.lad.mla_latent_decode_paged(self.q, self.pool, self.block_table, self.lens, self.gate, o=self.o,
                                         workspace=self.ws)
        if timer:
            timer.end("mla_latent_decode_paged")

    def mla_bytes(self):
        # the block table adds 4 bytes per page actually read
        return super().mla_bytes() + 4 * sum(-(-int(n) // self.page_size) for n in self.lens.tolist())

    def algorithmic_bytes(self):
        b = self.mla_bytes()
        return {"mla_latent_decode_paged": b, "step": b}


class MlaPagedRopeStep(MlaPagedStep):
    """The paged 16-sequence layer as an engine runs it: append each sequence's new row (latent +
    RoPE key turned to its position, mla_cache_append) and attend with the query's RoPE part
    turned inside the kernel (mla_latent_decode_paged_rope), both at position len - 1."""
    name = "mla_decode_b16_paged_rope"

    def __init__(self, lad, dev, rank, cfg: wl.MlaDecode | None = None):
        super().__init__(lad, dev, rank, cfg)
        B, s = self.cfg.B, self.cfg.seed
        self.c_kv = wl.normal_bf16((B, wl.D_LATENT), s, "mla_ckv", dev)
        self.k_pe = wl.normal_bf16((B, wl.D_ROPE), s, "mla_kpe", dev)
        self.pos = (self.lens - 1).contiguous()
        self.launches_per_step = 3
        self.dominant = "mla_latent_decode_paged_rope"
        self.config = dict(self.config, workload=self.name, rope="theta 6e6, rotate-half pairing, in-kernel")

    def run(self, timer=None):
        self.lad.mla_cache_append(self.c_kv, self.k_pe, self.pos, self.pool, block_table=self.block_table)
        if timer:
            timer.begin("mla_latent_decode_paged_rope")
        self.lad.mla_latent_decode_paged_rope(self.q, self.pos, self.pool, self.block_table, self.lens, self.gate,
                                              o=self.o, workspace=self.ws)
        if timer:
            timer.end("mla_latent_decode_paged_rope")

    def algorithmic_bytes(self):
        b = self.mla_bytes()
        append = self.cfg.B * (wl.D_LATENT * 2 + wl.D_ROPE * 2 + 4 + wl.D_ROW * 2 + 4)
        return {"mla_latent_decode_paged_rope": b, "step": b + append}


class MlaMultiStep(MlaDecodeStep):
    """The 16-sequence latent-attention workload as a multi-token verify step: 4 query tokens per
    sequence (a token and 3 drafts, the pages' MTP setting), token j attending the first
    len - 3 + j rows, through mla_latent_decode_multi. Algorithmic bytes count the cache once."""
    name = "mla_mtp_b16"
    T = 4

    def __init__(self, lad, dev, rank, cfg: wl.MlaDecode | None = None):
        super().__init__(lad, dev, rank, cfg)
        B, H, T, s = self.cfg.B, self.cfg.Hq, self.T, self.cfg.seed
        self.q = wl.normal_bf16((B, T, H, wl.D_ROW), s, "mla_q_mtp", dev)
        self.gate = wl.normal((B, T, H), s, "mla_gate_mtp", dev)
        self.o = torch.empty((B, T, H, wl.D_LATENT), device=dev, dtype=torch.bfloat16)
        self.ws = torch.empty(lad.mla_latent_decode_multi_workspace_size(B, T, H, wl.D_LATENT, 0), device=dev,
                              dtype=torch.uint8)
        self.h_q = self.q.cpu().pin_memory()
        self.h_gate = self.gate.cpu().pin_memory()
        self.h_o = torch.empty(self.o.shape, dtype=self.o.dtype).pin_memory()
        self.tokens_per_step = B * T
        self.launches_per_step = 3
        self.dominant = "mla_latent_decode_multi"
        self.config = dict(self.config, workload=self.name, query_tokens_per_sequence=T,
                           causal="token j attends rows 0 .. len - T + j")

    def run(self, timer=None):
        if timer:
            timer.begin("mla_latent_decode_multi")
        self.lad.mla_latent_decode_multi(self.q, self.cache, self.lens, self.gate, o=self.o, workspace=self.ws)
        if timer:
            timer.end("mla_latent_decode_multi")

    def mla_bytes(self):
        B, H, T = self.cfg.B, self.cfg.Hq, self.T
        return self.total_len * wl.D_ROW * 2 + B * T * H * (wl.D_ROW * 2 + 4 + wl.D_LATENT * 2) + B * 4

    def mla_flops(self):
        return self.T * super().mla_flops()

    def algorithmic_bytes(self):
        b = self.mla_bytes()
        return {"mla_latent_decode_multi": b, "step": b}


class MlaFp8Step(MlaDecodeStep):
    """The 16-sequence latent-attention workload over an FP8 (E4M3) cache with one fp32 scale,
    through mla_latent_decode_fp8; the cache holds half the bytes of the bf16 one."""
    name = "mla_decode_b16_fp8"

    def __init__(self, lad, dev, rank, cfg: wl.MlaDecode | None = None):
        super().__init__(lad, dev, rank, cfg)
        del self.cache
        torch.cuda.empty_cache()
        self.cache8 = wl.mla_fp8_cache(self.cfg, dev)
        self.kv_scale = wl.KV_SCALE_FP8
        self.dominant = "mla_latent_decode_fp8"
        self.config = dict(self.config, workload=self.name, cache_row="512 latent + 64 rope, E4M3 codes",
                           kv_scale=f"one fp32 scale per cache ({self.kv_scale})")

    def run(self, timer=None):
        if timer:
            timer.begin("mla_latent_decode_fp8")
        self.lad.mla_latent_decode_fp8(self.q, self.cache8, self.kv_scale, self.lens, self.gate, o=self.o,
                                       workspace=self.ws)
        if timer:
            timer.end("mla_latent_decode_fp8")

    def mla_bytes(self):
        B, Hq = self.cfg.B, self.cfg.Hq
        return self.total_len * wl.D_ROW + B * Hq * (wl.D_ROW * 2 + 4 + wl.D_LATENT * 2) + B * 4

    def algorithmic_bytes(self):
        b = self.mla_bytes()
        return {"mla_latent_decode_fp8": b, "step": b}


class MlaPagedRopeFp8Step(MlaFp8Step):
    """The engine step of mla_decode_b16_paged_rope over a pool of FP8 pages: mla_cache_append_fp8
    writes each sequence's new row at len - 1, then mla_latent_decode_paged_fp8 attends with the
    query's RoPE part turned in the kernel."""
    name = "mla_decode_b16_paged_rope_fp8"
    page_size = 64

    def __init__(self, lad, dev, rank, cfg: wl.MlaDecode | None = None):
        super().__init__(lad, dev, rank, cfg)
        self.pool, self.block_table = wl.paginate(self.cache8, self.lens, self.page_size, self.cfg.seed)
        del self.cache8
        torch.cuda.empty_cache()
        B, s = self.cfg.B, self.cfg.seed
        self.c_kv = wl.normal_bf16((B, wl.D_LATENT), s, "mla_ckv", dev)
        self.k_pe = wl.normal_bf16((B, wl.D_ROPE), s, "mla_kpe", dev)
        self.pos = (self.lens - 1).contiguous()
        self.launches_per_step = 3
        self.dominant = "mla_latent_decode_paged_fp8"
        self.config = dict(self.config, workload=self.name, rope="theta 6e6, rotate-half pairing, in-kernel",
                           paging=f"{self.page_size}-row pages, {self.pool.shape[0]} in a shuffled pool")

    def run(self, timer=None):
        self.lad.mla_cache_append_fp8(self.c_kv, self.k_pe, self.pos, self.pool, self.kv_scale,
                                      block_table=self.block_table)
        if timer:
            timer.begin("mla_latent_decode_paged_fp8")
        self.lad.mla_latent_decode_paged_fp8(self.q, self.pool, self.kv_scale, self.block_table, self.lens,
                                             positions=self.pos, gate_logits=self.gate, o=self.o, workspace=self.ws)
        if timer:
            timer.end("mla_latent_decode_paged_fp8")

    def mla_bytes(self):
        return super().mla_bytes() + 4 * sum(-(-int(n) // self.page_size) for n in self.lens.tolist())

    def algorithmic_bytes(self):
        b = self.mla_bytes()
        append = self.cfg.B * (wl.D_LATENT * 2 + wl.D_ROPE * 2 + 4 + wl.D_ROW + 4)
        return {"mla_latent_decode_paged_fp8": b, "step": b + append}


class HybridStep(Step):
    name = "hybrid_8layer_1m"

    def __init__(self, lad, dev, rank, B=8, ctx=1_000_000, kda_layers=7):
        seed = 1238 + 1000 * rank
        self.kda = [_KdaLayer(lad, B, seed, dev, tag=f"L{i}.") for i in range(kda_layers)]
        # each layer's kernel follows another layer's (or the MLA combine), never its own state's
        # previous step, so its state reads may start while that kernel drains
        for layer in self.kda:
            layer.overlap = True
        self.mla = MlaDecodeStep(lad, dev, rank, wl.MlaDecode("mla", B=B, seed=seed, fixed_len=ctx))
        self.tokens_per_step = B
        self.launches_per_step = (1 if _KdaLayer.fused else 2) * kda_layers + self.mla.launches_per_step
        self.dominant = "mla_latent_decode"
        self.dominant_units = lambda: self.mla.total_len
        self.config = {"workload": self.name, "batch_per_gpu": B, "layers": f"{kda_layers} KDA + 1 gated MLA",
                       "kda_path": ("fused conv+step" if _KdaLayer.fused else "conv, then step")
                       + ", programmatic dependent launches (state reads overlap the previous layer's drain)",
                       "mla_context": ctx, "heads": H, "head_dim": D,
                       "l2": "inputs larger than L2 (9.2 GB latent cache + 235 MB KDA state per step)"}

    def run(self, timer=None):
        # the seven KDA layers are timed as one bracket (short kernels: see KernelTimer)
        kname = "kda_conv_decode_step" if _KdaLayer.fused else None
        if timer and kname:
            timer.begin(kname, count=len(self.kda))
        for layer in self.kda:
            layer.run(None if kname else timer)
        if timer and kname:
            timer.end(kname)
        self.mla.run(timer)

    def _io_names(self, part):
        return ("q", "gate", "o") if part is self.mla else ("x", "alpha", "beta", "o")

    def run_e2e(self):
        # A serving loop: two sets of device input / output buffers, so that the next step's token
        # inputs go up on one copy stream while this step computes, and this step's outputs come
        # back on another while the next one computes. Every step still copies its own
        # inputs in and its own outputs out. The state and conv tails stay on the device, updated
        # in order by the compute stream.
        cur = torch.cuda.current_stream()
        parts = (*self.kda, self.mla)
        if not hasattr(self, "_copy_stream"):
            self._copy_stream = torch.cuda.Stream()   # inputs up
            self._back_stream = torch.cuda.Stream()   # outputs back
            self._sets = [{id(pt): {n: getattr(pt, n) for n in self._io_names(pt)} for pt in parts}]
            self._sets.append({id(pt): {n: torch.empty_like(getattr(pt, n)) for n in self._io_names(pt)}
                               for pt in parts})
            self._free = [None, None]  # copy-stream event: the set's last outputs are back on the host
            self._parity = 0
        cs, p = self._copy_stream, self._parity
        self._parity ^= 1
        for pt in parts:
            for n, t in self._sets[p][id(pt)].items():
                setattr(pt, n, t)
        with torch.cuda.stream(cs):
            if self._free[p] is not None:
                cs.wait_event(self._free[p])
            for pt in parts:
                pt.h2d()
            landed = torch.cuda.Event()
            landed.record(cs)
        # one wait for the whole step's inputs (they went up while the step before it ran), so
        # that the layers' kernels follow one another on the stream with nothing in between and
        # each KDA launch overlaps the one before it
        cur.wait_event(landed)
        for pt in parts:
            pt.run()
        done = torch.cuda.Event()
        done.record(cur)
        bs = self._back_stream
        with torch.cuda.stream(bs):
            bs.wait_event(done)
            for pt in parts:
                pt.d2h()
            self._free[p] = torch.cuda.Event()
            self._free[p].record(bs)

    def e2e_drain(self):
        """The compute stream waits for the outputs still on their way back."""
        if hasattr(self, "_back_stream"):
            torch.cuda.current_stream().wait_stream(self._back_stream)

    def e2e_bytes(self):
        hb = sum(layer.h2d_bytes() for layer in self.kda) + self.mla.e2e_bytes()[0]
        db = sum(layer.d2h_bytes() for layer in self.kda) + self.mla.e2e_bytes()[1]
        return hb, db

    def algorithmic_bytes(self):
        B = self.kda[0].B
        n = len(self.kda)
        kd, kc, m = _KdaLayer.bytes_decode(B), _KdaLayer.bytes_conv(B), self.mla.mla_bytes()
        kf = _KdaLayer.bytes_fused(B)
        return {"kda_decode_step": kd, "kda_conv_update": kc, "kda_conv_decode_step": kf, "mla_latent_decode": m,
                "step": n * (kf if _KdaLayer.fused else kd + kc) + m}


class PrefillStep(Step):
    name = "kda_prefill_32k"

    # fp16 operand tiles (kind::f16): the tensor floor (~3.8e11 flop at the f16 peak) sits below the
    # HBM floor (~3.2 GB at the copy peak), so the roofline is HBM's; the tensor view is reported beside it
    dominant_bound = "hbm"

    def __init__(self, lad, dev, rank, cfg: wl.KdaScan | None = None):
        cfg = cfg or wl.KdaScan("prefill", B=1, H=64, T=32768, chunk=64, seed=1237 + 1000 * rank)
        self.lad, self.cfg = lad, cfg
        inp = wl.kda_scan_inputs(cfg, dev)
        self.q, self.k, self.v = inp["q"], inp["k"], inp["v"]
        self.alpha, self.beta, self.S0 = inp["alpha"], inp["beta"], inp["S0"]
        self.S = self.S0.clone()
        self.o = torch.empty_like(self.v)
        self.ws = torch.empty(max(1, lad.kda_prefill_workspace_size(cfg.B, cfg.T, cfg.H, D, D, cfg.chunk)),
                              device=dev, dtype=torch.uint8)
        self.h_in = [t.cpu().pin_memory() for t in (self.q, self.k, self.v, self.alpha, self.beta)]
        self.h_o = torch.empty(self.o.shape, dtype=self.o.dtype).pin_memory()
        self.tokens_per_step = cfg.B * cfg.T
        # the two-kernel path (a workspace is given): segments of up to 128 chunks, the last one 32
        # when there are several; the first segment's prep is one launch, every later one two (beside
        # the previous chain, and behind it), and each segment has one chain launch
        nch = math.ceil(cfg.T / cfg.chunk)
        nsegs = 1 if nch <= 128 else math.ceil((nch - 32) / 128) + 1
        self.launches_per_step = 2 + 3 * (nsegs - 1)
        self.dominant = "kda_prefill_chunked"
        self.config = {"workload": self.name, "batch_per_gpu": cfg.B, "seq_len": cfg.T, "heads": cfg.H,
                       "chunk": cfg.chunk, "l2": f"inputs larger than L2 ({self.algorithmic_bytes()['step'] / 1e9:.2f} GB per step)"}

    def run(self, timer=None):
        if timer:
            timer.begin("kda_prefill_chunked")
        self.S.copy_(self.S0)
        self.lad.kda_prefill_chunked(self.q, self.k, self.v, self.alpha, self.beta, self.S, o=self.o,
                                     chunk=self.cfg.chunk, workspace=self.ws)
        if timer:
            timer.end("kda_prefill_chunked")

    def run_e2e(self):
        for d, h in zip((self.q, self.k, self.v, self.alpha, self.beta), self.h_in):
            d.copy_(h, non_blocking=True)
        self.run()
        self.h_o.copy_(self.o, non_blocking=True)

    def e2e_bytes(self):
        return sum(t.numel() * t.element_size() for t in self.h_in), self.h_o.numel() * 2

    def dominant_units(self):
        return self.cfg.B * self.cfg.T * self.cfg.H

    def algorithmic_bytes(self):
        c = self.cfg
        n = c.B * c.T * c.H
        b = n * (3 * D * 2 + D * 4 + 4 + D * 2) + 2 * c.B * c.H * D * D * 4
        return {"kda_prefill_chunked": b, "step": b}

    def flops(self):
        c = self.cfg
        chunks = c.B * c.H * math.ceil(c.T / c.chunk)
        C = c.chunk
        # multiply-adds per chunk-head: [Qt; Kt] Kh^T (2 C C D), W = Tb Kt (C C D), U' = Tb V (C C D),
        # X = W S0 (C D D), O = Qt S0 (C D D) + lower(Qt Kh^T) U (C C D), S += Kh^T U (D D C)
        # (the single kernel forms Tb (Kt S0) instead of (Tb Kt) S0: the same count)
        per_chunk = 2 * (2 * C * C * D + C * C * D + C * C * D + C * D * D + C * D * D + C * C * D + D * D * C)
        return chunks * per_chunk


WORKLOADS = {
    "hybrid_8layer_1m": HybridStep,
    "kda_decode_b64": KdaDecodeStep,
    "kda_decode_b64_gated": KdaGatedStep,
    "kda_mtp_b64": KdaMultiStep,
    "mla_decode_b16": MlaDecodeStep,
    "mla_decode_b16_paged": MlaPagedStep,
    "mla_decode_b16_paged_rope": MlaPagedRopeStep,
    "mla_mtp_b16": MlaMultiStep,
    "mla_decode_b16_fp8": MlaFp8Step,
    "mla_decode_b16_paged_rope_fp8": MlaPagedRopeFp8Step,
    "kda_prefill_32k": PrefillStep,
}


class KernelTimer:
    """CUDA events around each launch of named kernels, on the current (launching) stream. A pair
    may bracket `count` back-to-back launches of the same kernel (then it is timed per launch as
    the bracket's time / count), which keeps the events' own cost out of short kernels."""

    def __init__(self):
        self.pairs: dict[str, list] = {}

    def begin(self, name, count: int = 1):
        e = torch.cuda.Event(enable_timing=True)
        e.record()
        self.pairs.setdefault(name, []).append([e, None, count])

    def end(self, name):
        e = torch.cuda.Event(enable_timing=True)
        e.record()
        self.pairs[name][-1][1] = e

    def mean_ms(self, name) -> float | None:
        ps = self.pairs.get(name)
        if not ps:
            return None
        return sum(a.elapsed_time(b) for a, b, _ in ps) / sum(n for _, _, n in ps)


# ---------------------------------------------------------------------------------------------
# CPU oracle timing (the reference arm and the cpu_baseline key)
# ---------------------------------------------------------------------------------------------

class OracleSample:
    """One bounded sample of a workload step for the fp64 oracle on `nth` host threads.

    The sample is a list of parts, each an oracle call over a subset of the step's units (some
    of a layer's sequences, some heads over a context) with the factor that scales its time to
    the whole step; the sample's size follows `nth`, so one thread runs a proportionally smaller
    sample. run() returns the estimated seconds of one whole workload step."""

    def __init__(self, workload: str, nth: int):
        import oracle
        self.oracle, self.nth = oracle, nth
        rng = np.random.default_rng(0)
        self.parts: list[tuple] = []   # (callable, factor)
        desc = []

        def kda_layer(B):
            Bs = min(B, max(1, nth))
            x = rng.standard_normal((Bs, 3 * H * D))
            tail = rng.standard_normal((Bs, 3, 3 * H * D))
            w = 0.5 * rng.standard_normal((3 * H * D, 4))
            S = 0.02 * rng.standard_normal((Bs, H, D, D))
            a = np.full((Bs, 1, H, D), 0.9)
            b = np.full((Bs, 1, H), 0.5)

            def run():
                y, _ = oracle.short_conv_step(x, tail, w, None, True)
                qn = oracle.l2norm(y[:, : H * D].reshape(Bs, 1, H, D))
                kn = oracle.l2norm(y[:, H * D: 2 * H * D].reshape(Bs, 1, H, D))
                oracle.kda_recurrent(qn, kn, y[:, 2 * H * D:].reshape(Bs, 1, H, D), a, b, S.copy(), nthreads=nth)
            return run, B / Bs, f"{Bs} of {B} sequences x 64 heads, one token"

        def mla(lens, fp8=False):
            # (sequence, head) units: `units` heads of the longest sequence over its whole context
            L = int(max(lens))
            units = min(max(1, nth), H)
            qs = rng.standard_normal((1, units, wl.D_ROW))
            ln = np.array([L], np.int32)
            if fp8:
                codes = rng.integers(0, 0x7F, (1, L, wl.D_ROW), dtype=np.uint8)

                def run():
                    oracle.mla_decode_fp8(qs, codes, wl.KV_SCALE_FP8, ln, None, nthreads=nth)
            else:
                cache = (rng.standard_normal((1, L, wl.D_ROW)).astype(np.float32).view(np.uint32) >> 16).astype(
                    np.uint16)

                def run():
                    oracle.mla_decode(qs, cache, ln, None, nthreads=nth)
            return run, H * float(sum(lens)) / (units * L), f"{units} heads x {L} cached tokens of 1 sequence"

        if workload in ("kda_decode_b64", "kda_decode_b64_gated"):
            f, k, d = kda_layer(64)
            self.parts.append((f, k))
            desc.append(d)
        elif workload == "kda_mtp_b64":
            Bs = min(64, max(1, nth))
            q = rng.standard_normal((Bs, 4, H, D))
            S = 0.02 * rng.standard_normal((Bs, H, D, D))
            a = np.full((Bs, 4, H, D), 0.9)
            b = np.full((Bs, 4, H), 0.5)
            self.parts.append((lambda: oracle.kda_recurrent(q, q, q, a, b, S.copy(), nthreads=nth), 64 / Bs))
            desc.append(f"{Bs} of 64 sequences x 64 heads x 4 tokens")
        elif workload in ("mla_decode_b16", "mla_decode_b16_paged", "mla_decode_b16_paged_rope",
                          "mla_decode_b16_fp8", "mla_decode_b16_paged_rope_fp8"):
            lens = wl.mla_seq_lens(wl.MlaDecode("mla", B=16, seed=1236)).tolist()
            f, k, d = mla(lens, fp8=workload.endswith("fp8"))
            self.parts.append((f, k))
            desc.append(d)
        elif workload == "mla_mtp_b16":  # four query tokens: four attentions over (nearly) the rows
            lens = wl.mla_seq_lens(wl.MlaDecode("mla", B=16, seed=1236)).tolist()
            f, k, d = mla(lens)
            self.parts.append((f, 4 * k))
            desc.append(d + ", x4 query tokens")
        elif workload == "hybrid_8layer_1m":
            f, k, d1 = kda_layer(8)
            self.parts.append((f, 7 * k))
            g, m, d2 = mla([1_000_000] * 8)
            self.parts.append((g, m))
            desc.append(f"KDA layer: {d1} (x7 layers); MLA: {d2}")
        elif workload == "kda_prefill_32k":
            T, Hs = 1024, min(max(1, nth), H)
            q = rng.standard_normal((1, T, Hs, D))
            a = np.full((1, T, Hs, D), 0.95)
            b = np.full((1, T, Hs), 0.5)
            S = np.zeros((1, Hs, D, D))
            self.parts.append((lambda: oracle.kda_recurrent(q, q, q, a, b, S.copy(), nthreads=nth),
                               (32768 / T) * (64 / Hs)))
            desc.append(f"{Hs} heads x {T} tokens")
        else:
            raise ValueError(workload)
        self.sample = "; ".join(desc) + "; scaled to the whole step"

    def run(self) -> float:
        est = 0.0
        for f, k in self.parts:
            t0 = time.perf_counter()
            f()
            est += (time.perf_counter() - t0) * k
        return est


def cpu_oracle_rate(workload: str, nth: int | None = None, repeats: int = 3) -> dict:
    """The fp64 oracle's rate (tokens/s of the whole workload step) from the median of `repeats`
    timed samples after one untimed one, on `nth` threads (default: all host cores)."""
    import oracle
    nth = oracle.max_threads() if nth is None else nth
    smp = OracleSample(workload, nth)
    smp.run()
    est = [smp.run() for _ in range(repeats)]
    med = statistics.median(est)
    return {"value": _tokens(workload) / med, "unit": "tokens/s", "cores": nth, "kind": "oracle",
            "sample": smp.sample, "repeats": repeats,
            "spread": round((max(est) - min(est)) / med, 4)}


def cpu_baseline(workload: str) -> dict:
    """The all-core oracle rate, with the single-thread rate beside it."""
    cb = cpu_oracle_rate(workload)
    one = cpu_oracle_rate(workload, nth=1)
    cb["single_thread"] = {"value": one["value"], "unit": one["unit"], "sample": one["sample"],
                           "repeats": one["repeats"]}
    return cb


# ---------------------------------------------------------------------------------------------

def run_reference(args, rank, world):
    """The oracle as the reference arm: W untimed and K timed steps, each step one bounded sample
    of the workload (OracleSample) on all host cores; ms_per_step is the median wall time of a
    sample, value the tokens/s of the whole workload step the samples estimate."""
    if rank != 0:
        return 0
    import oracle
    nth = oracle.max_threads()
    smp = OracleSample(args.workload, nth)
    for _ in range(args.warmup):
        smp.run()
    wall, est = [], []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        est.append(smp.run())
        wall.append(time.perf_counter() - t0)
    step_s = statistics.median(est)
    value = _tokens(args.workload) / step_s
    one = cpu_oracle_rate(args.workload, nth=1)
    cb = {"value": value, "unit": "tokens/s", "cores": nth, "kind": "oracle", "sample": smp.sample,
          "repeats": args.steps, "single_thread": {"value": one["value"], "unit": one["unit"],
                                                    "sample": one["sample"], "repeats": one["repeats"]}}
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * statistics.median(wall),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, "implementation": "fp64 CPU oracle (plain C, OpenMP over heads)",
                       "step": "one bounded sample of the workload step (see cpu_baseline.sample); value is the "
                               "whole step's tokens over the step time the samples estimate (median)",
                       "estimated_ms_per_workload_step": 1000.0 * step_s},
            "cpu_baseline": cb,
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def _tokens(workload):
    return {"hybrid_8layer_1m": 8, "kda_decode_b64": 64, "kda_decode_b64_gated": 64, "kda_mtp_b64": 256, "mla_decode_b16": 16,
            "mla_decode_b16_paged": 16, "mla_decode_b16_paged_rope": 16, "mla_decode_b16_fp8": 16,
            "mla_decode_b16_paged_rope_fp8": 16, "mla_mtp_b16": 64, "kda_prefill_32k": 32768}[workload]


def time_device(step, steps: int, warmup: int, local: int, dev):
    """W untimed steps, then device events around exactly K steps (per-kernel events inside), with
    the SM clock sampled meanwhile; the step time is the max over ranks."""
    for _ in range(warmup):
        step.run()
    torch.cuda.synchronize()
    barrier(local)
    timer = KernelTimer()
    clocks = ClockSampler(physical_gpu_index(local))
    clocks.start()
    time.sleep(0.3)
    torch.cuda.synchronize()
    barrier(local)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(steps):
        step.run(timer)
    t1.record()
    torch.cuda.synchronize()
    barrier(local)
    clk = clocks.stop()
    ms = max_over_ranks(t0.elapsed_time(t1) / steps, dev)
    return ms, timer, clk


# configs 1-3 of the workload list, timed after the headline in the same process: the single
# KDA decode layer (64 x 64 heads), the 16-sequence MLA layer, and the 32K-token prefill
PER_CONFIG = (("kda_decode_b64", "config 1: KDA decode layer, 64 sequences x 64 heads, conv fused"),
              ("mla_decode_b16", "config 2: gated MLA decode, 16 sequences, contexts uniform in [8192, 131072]"),
              ("kda_prefill_32k", "config 3: KDA chunked prefill, 1 x 32768 tokens x 64 heads, chunk 64"))


def per_config_lines(lad, dev, rank, local, steps: int, warmup: int, peaks: dict) -> dict:
    out = {}
    for name, what in PER_CONFIG:
        step = WORKLOADS[name](lad, dev, rank)
        torch.cuda.synchronize()
        ms, timer, clk = time_device(step, steps, warmup, local, dev)
        km = timer.mean_ms(step.dominant)
        ab = step.algorithmic_bytes()
        gbs = ab[step.dominant] / (km / 1000.0) / 1e9
        e = {"what": what, "kernel": step.dominant, "ms_per_step": round(ms, 4), "ms_per_launch": round(km, 4),
             "tokens_per_s": step.tokens_per_step / (ms / 1000.0), "gb_s": round(gbs, 1),
             "frac_of_measured_hbm": round(gbs / peaks["hbm_gbs"], 4), "steps": steps, "warmup": warmup,
             "clocks": {"sm_mhz": clk["sm_mhz"], "sm_max_mhz": clk["sm_max_mhz"], "reasons": clk["reasons"]}}
        if isinstance(step, PrefillStep):
            tf = step.flops() / (km / 1000.0) / 1e12
            e.update({"tflop_s": round(tf, 1), "frac_of_f16_tensor_peak": round(tf / peaks["bf16_tflops"], 4)})
        if isinstance(step, MlaDecodeStep):
            e["mma_tflop_s"] = round(step.mla_flops() / (km / 1000.0) / 1e12, 1)
        out[name] = e
        del step
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
    return out


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="lad", choices=["lad", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--seq-len", type=int, default=32768, help="tokens of the kda_prefill_32k workload")
    ap.add_argument("--unfused-conv", action="store_true",
                    help="KDA layers as kda_conv_update + kda_decode_step instead of kda_conv_decode_step")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the per_config timings of configs 1-3 after the default workload")
    args = ap.parse_args(argv)
    _KdaLayer.fused = not args.unfused_conv
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    rank, world, local = dist_env()
    if args.impl == "reference":
        return run_reference(args, rank, world)

    import latent_attention_decode_b200 as lad
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    if args.workload == "kda_prefill_32k":
        step = PrefillStep(lad, dev, rank, wl.KdaScan("prefill", B=1, H=64, T=args.seq_len, chunk=64,
                                                      seed=1237 + 1000 * rank))
    else:
        step = WORKLOADS[args.workload](lad, dev, rank)
    torch.cuda.synchronize()

    ms, timer, clk = time_device(step, args.steps, args.warmup, local, dev)

    # end to end through the public API: pinned host inputs in, outputs back, every step
    for _ in range(3):
        step.run_e2e()
    torch.cuda.synchronize()
    barrier(local)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        step.run_e2e()
    if hasattr(step, "e2e_drain"):
        step.e2e_drain()
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, dev)
    barrier(local)

    tokens = sum_over_ranks(float(step.tokens_per_step), dev)
    value = tokens / (ms / 1000.0)
    peaks = measured_peaks()
    ab = step.algorithmic_bytes()
    dom_ms = timer.mean_ms(step.dominant)
    achieved = ab[step.dominant] / (dom_ms / 1000.0) / 1e9
    per_type = {}
    for kname in ("kda_conv_decode_step", "kda_conv_decode_step_gated", "kda_decode_step", "kda_decode_multi",
                  "mla_latent_decode",
                  "mla_latent_decode_paged", "mla_latent_decode_paged_rope", "mla_latent_decode_fp8",
                  "mla_latent_decode_paged_fp8", "mla_latent_decode_multi", "kda_prefill_chunked"):
        km = timer.mean_ms(kname)
        if km is not None and kname in ab:
            gbs = ab[kname] / (km / 1000.0) / 1e9
            per_type[kname] = {"ms_per_launch": round(km, 4), "gb_s": round(gbs, 1),
                               "frac_of_measured_hbm": round(gbs / peaks["hbm_gbs"], 4),
                               "frac_of_8tbs_spec": round(gbs / 8000.0, 4)}
    if isinstance(step, PrefillStep) and dom_ms:
        tf = step.flops() / (dom_ms / 1000.0) / 1e12
        per_type["kda_prefill_chunked"]["tflop_s"] = round(tf, 1)
        per_type["kda_prefill_chunked"]["frac_of_f16_tensor_peak"] = round(tf / peaks["bf16_tflops"], 4)
    if isinstance(step, (MlaDecodeStep, HybridStep)):
        m = step if isinstance(step, MlaDecodeStep) else step.mla
        kname = m.dominant
        km = timer.mean_ms(kname)
        per_type[kname]["mma_tflop_s"] = round(m.mla_flops() / (km / 1000.0) / 1e12, 1)

    line = None
    if rank == 0:
        hb, db = step.e2e_bytes()
        traffic = kernel_traffic(step.dominant, step.dominant_units())
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": ("e4m3 cache widened to bf16, bf16 query, fp32 accumulation"
                                           if args.workload.endswith("fp8") else
                                           "bf16 inputs, fp32 state and accumulation"), "data": "synthetic",
            "config": {**step.config, "global_batch": int(round(tokens)) if not isinstance(step, PrefillStep)
                       else world * step.cfg.B, "parallelism": f"sequence-sharded x{world}, no exchange"},
            "per_layer_type": per_type,
            "step_gb_s": ab["step"] / (ms / 1000.0) / 1e9,
            "roofline": {"kernel": step.dominant, "bound": "hbm", "achieved": achieved,
                         "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                         "traffic": traffic["bytes"] if traffic else None,
                         "traffic_source": traffic, "peak_source": f"{peaks['source']} hbm_gbs (copy)",
                         "algorithmic_bytes_per_launch": ab[step.dominant]},
            "cpu_baseline": None,
            "e2e": {"value": tokens / (e2e_ms / 1000.0), "unit": "tokens/s", "h2d_bytes_per_step": hb * world,
                    "d2h_bytes_per_step": db * world},
            "gpu_launches": step.launches_per_step * args.steps,
            "clocks": {"sm_mhz": clk["sm_mhz"], "sm_max_mhz": clk["sm_max_mhz"], "reasons": clk["reasons"]},
        }
        if isinstance(step, PrefillStep):
            # the f16 tensor view of the same launch (kind::f16 runs at the bf16 rate): the measured
            # bf16 burst peak, the method's algorithmic flops
            tf = step.flops() / (dom_ms / 1000.0) / 1e12
            line["roofline_tensor"] = {"kernel": step.dominant, "bound": "tensor", "achieved": tf,
                                       "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                                       "frac": tf / peaks["bf16_tflops"],
                                       "peak_source": f"{peaks['source']} bf16_tflops (burst; f16 runs at the same rate)",
                                       "algorithmic_flops_per_launch": step.flops(),
                                       "tensor_pipe_active_pct": traffic.get("tensor_pipe_active_pct") if traffic else None}

    # configs 1-3 (single GPU), after the headline, when the default workload runs alone; their
    # launches are not counted in gpu_launches, which covers the headline's timed region only
    if world == 1 and args.workload == DEFAULT_WORKLOAD and not args.no_per_config:
        del step
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        line["per_config"] = per_config_lines(lad, dev, rank, local, min(args.steps, 10), args.warmup, peaks)

    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(args.workload)
        print(json.dumps(line), flush=True)

    if world > 1:
        import torch.distributed as dist
        barrier(local)
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
