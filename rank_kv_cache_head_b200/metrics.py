"""Measurement helpers: algorithmic byte counts, an nvidia-smi clock sampler, and the
max-over-ranks aggregation used by the benchmark.

Algorithmic bytes of one decode-attention call (one layer, one new token per row):
  latent  = sum_b L_b * H_kv * 2 * r * bytes(latent)      (Z_K and Z_V, valid rows)
  scales  = sum_b L_b * H_kv * 2 * 4                      (quantised latents only)
  factors = 2 * H_kv * r * d * bytes(io)                  (B_K, B_V once)
  q, out  = B * H_q * d * bytes(io) each
Split partials and the workspace are not counted. The split kernel's share is
everything but ``out`` (the merge kernel writes the output).
"""
from __future__ import annotations

import statistics
import subprocess
import threading
import time
from typing import Optional

import numpy as np

_BYTES = {"f32": 4, "bf16": 2, "i8": 1, "e4m3": 1}


def step_bytes(wl, seqlens, factor_sets: int = 1) -> dict:
    tok_heads = int(np.sum(np.asarray(seqlens, np.int64))) * wl.n_kv_heads
    quant = wl.latent_dtype in ("i8", "e4m3")
    latent = tok_heads * 2 * wl.rank * _BYTES[wl.latent_dtype]
    scales = tok_heads * 2 * 4 if quant else 0
    io = _BYTES[wl.io_dtype]
    factors = factor_sets * 2 * wl.n_kv_heads * wl.rank * wl.d_head * io
    q = wl.batch * wl.n_q_heads * wl.d_head * io
    out = q
    total = latent + scales + factors + q + out
    return {"latent": latent, "scales": scales, "factors": factors, "q": q, "out": out,
            "total": total, "split_kernel": total - out, "token_heads": tok_heads}


class ClockSampler:
    """Samples SM clocks, power and throttle reasons with nvidia-smi while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index, period_ms: int = 50):
        self.gpu_index = gpu_index
        self.period_ms = period_ms
        self.samples = []   # (t, sm_mhz, max_mhz, power_w, active_mask, hw, hwt, swt, swpc)
        self.proc: Optional[subprocess.Popen] = None
        self.thread: Optional[threading.Thread] = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 f"-lms={self.period_ms}", f"-i={self.gpu_index}"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return self
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        return self

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                self.samples.append((time.perf_counter(), float(parts[1]), float(parts[2]),
                                     float(parts[3]) if parts[3] not in ("[N/A]", "N/A") else 0.0,
                                     parts[4], *parts[5:9]))
            except ValueError:
                continue

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)

    def summary(self, t0: float, t1: float) -> dict:
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        window = "timed"
        if len(inside) < 3:
            inside = self.samples
            window = "whole run (timed region shorter than the sampling period)"
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({n for s in inside for n, v in zip(names, s[5:9]) if v == "Active"})
        return {"sm_mhz": statistics.median(s[1] for s in inside),
                "sm_max_mhz": max(s[2] for s in inside),
                "power_w_max": max(s[3] for s in inside),
                "samples": len(inside), "window": window, "reasons": reasons}


def max_over_ranks(value: float, device=None) -> float:
    """Max of a float over all ranks (identity without torch.distributed)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64,
                     device=device if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64,
                     device=device if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())
