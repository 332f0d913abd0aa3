"""Seeded synthetic workloads for low-rank KV-cache decode attention.

This module only draws inputs. It holds none of the arithmetic of the decode path
(no reconstruction, no softmax, no quantiser): the oracle and the CUDA path both
consume what it returns, so it is the one piece of code they share.

The five workloads are synthetic stand-ins for the vision-language and LLaMA decode
benchmarks the low-rank KV-cache pages report on (their models, weights and datasets
are not available here):

  tiny-fp32       batch 1, 4 q heads = 4 KV heads, d_head 64, rank 16, seq 256, fp32
  vlm7b-bf16      batch 8, 32/32 heads, d_head 128, rank 32, seq 4096, bf16
                  (first 576 positions are tagged "visual"; same distribution)
  gqa-ragged-bf16 batch 64, 32/8 heads, d_head 128, rank 48, seq_len_b ~ U[128, 4096]
  longvideo-bf16  batch 4, 32/8 heads, d_head 128, rank 64, seq 32768,
                  1% of positions per row scaled x8 (outlier tokens)
  quant-i8 / quant-e4m3
                  batch 32, 32/8 heads, d_head 128, rank 32, seq 8192, latents
                  stored as int8 or fp8-e4m3 codes with one fp32 scale per token

Recipe (all draws from numpy PCG64 with the workload's seed, in float64, then cast to
the stored dtype with torch's round-to-nearest-even casts):
  * Z_K, Z_V ~ N(0, 1) per element; outlier rows (long-video) multiplied by 8, the same
    positions for every KV head and for both Z_K and Z_V.
  * B_K, B_V = diag(sigma) . Q^T where Q (d x r) is the QR factor of a Gaussian d x r
    matrix with the sign of diag(R) made positive (orthonormal rows); sigma_i for
    i = 1..r is 0.9^i, 0.95^i or i^-0.5.
  * q ~ N(0, 1).
  * Quantised latents: the codes are drawn directly, not produced by a quantiser:
    int8 codes are a Gaussian with std 127/3, rounded and clipped to [-127, 127];
    e4m3 codes are torch's cast of a Gaussian with std 448/4 clipped to [-448, 448].
    The per-token scale is 3/127 (int8) or 4/448 (e4m3) times U(0.8, 1.2), drawn per
    (batch, KV head, token), so code x scale is roughly N(0, 1) like the bf16 latents.
  * Cache rows at positions >= seq_len_b are zero, or NaN / 1e30 when ``poison`` is
    set (they must never influence a result).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    n_q_heads: int
    n_kv_heads: int
    d_head: int
    rank: int
    seq_len: int                 # longest sequence (every row unless ragged)
    io_dtype: str                # "f32" | "bf16": q, out, B_K, B_V
    latent_dtype: str            # "f32" | "bf16" | "i8" | "e4m3": Z_K, Z_V
    sigma: tuple                 # ("geom", base) or ("pow", exponent)
    ragged_min: Optional[int] = None  # seq_len_b ~ U[ragged_min, seq_len]
    outlier_frac: float = 0.0
    outlier_scale: float = 1.0
    visual_prefix: int = 0       # positions tagged visual (no structural effect)
    seed: int = 0

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny-fp32": Workload("tiny-fp32", 1, 4, 4, 64, 16, 256, "f32", "f32",
                          ("geom", 0.9), seed=1001),
    "vlm7b-bf16": Workload("vlm7b-bf16", 8, 32, 32, 128, 32, 4096, "bf16", "bf16",
                           ("pow", -0.5), visual_prefix=576, seed=1002),
    "gqa-ragged-bf16": Workload("gqa-ragged-bf16", 64, 32, 8, 128, 48, 4096, "bf16", "bf16",
                                ("geom", 0.95), ragged_min=128, seed=1003),
    "longvideo-bf16": Workload("longvideo-bf16", 4, 32, 8, 128, 64, 32768, "bf16", "bf16",
                               ("pow", -0.5), outlier_frac=0.01, outlier_scale=8.0,
                               seed=1004),
    "quant-i8": Workload("quant-i8", 32, 32, 8, 128, 32, 8192, "bf16", "i8",
                         ("geom", 0.9), seed=1005),
    "quant-e4m3": Workload("quant-e4m3", 32, 32, 8, 128, 32, 8192, "bf16", "e4m3",
                           ("geom", 0.9), seed=1006),
}

_TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}


def sigmas(wl: Workload) -> np.ndarray:
    i = np.arange(1, wl.rank + 1, dtype=np.float64)
    kind, p = wl.sigma
    if kind == "geom":
        return p ** i
    if kind == "pow":
        return i ** p
    raise ValueError(kind)


def _orthonormal_rows(rng: np.random.Generator, r: int, d: int) -> np.ndarray:
    a = rng.standard_normal((d, r))
    qm, rm = np.linalg.qr(a)
    qm = qm * np.sign(np.diag(rm))[None, :]
    return qm.T  # r x d, orthonormal rows


def seqlens_for(wl: Workload, rng: Optional[np.random.Generator] = None) -> np.ndarray:
    if wl.ragged_min is None:
        return np.full(wl.batch, wl.seq_len, dtype=np.int32)
    rng = rng or np.random.default_rng(wl.seed + 7)
    return rng.integers(wl.ragged_min, wl.seq_len + 1, size=wl.batch).astype(np.int32)


def make_inputs(wl: Workload, capacity: Optional[int] = None, poison: Optional[str] = None,
                seqlens: Optional[np.ndarray] = None) -> dict:
    """Draw one decode step's inputs in their stored dtypes (CPU torch tensors).

    Returns q [B][Hq][d], ZK/ZV [B][Hkv][L_cap][r], ZK_scale/ZV_scale [B][Hkv][L_cap]
    (fp32, quantised latents only, else None), BK/BV [Hkv][r][d], seqlens [B] int32.
    ``poison`` = None | "nan" | "big" fills the cache rows past seq_len_b.
    """
    B, Hq, Hkv, d, r = wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.d_head, wl.rank
    rng = np.random.default_rng(np.random.PCG64(wl.seed))
    if seqlens is None:
        seqlens = seqlens_for(wl, np.random.default_rng(wl.seed + 7))
    seqlens = np.asarray(seqlens, dtype=np.int32)
    L_cap = int(capacity if capacity is not None else max(int(seqlens.max()), 1))
    if int(seqlens.max()) > L_cap:
        raise ValueError("capacity below the longest sequence")

    sig = sigmas(wl)
    BK = np.stack([sig[:, None] * _orthonormal_rows(rng, r, d) for _ in range(Hkv)])
    BV = np.stack([sig[:, None] * _orthonormal_rows(rng, r, d) for _ in range(Hkv)])
    q = rng.standard_normal((B, Hq, d))

    io_t = _TORCH_DTYPE[wl.io_dtype]
    out = {
        "q": torch.from_numpy(np.ascontiguousarray(q)).to(io_t).contiguous(),
        "BK": torch.from_numpy(np.ascontiguousarray(BK)).to(io_t).contiguous(),
        "BV": torch.from_numpy(np.ascontiguousarray(BV)).to(io_t).contiguous(),
        "seqlens": torch.from_numpy(seqlens.copy()),
    }

    lat = wl.latent_dtype
    if lat in ("f32", "bf16"):
        zt = _TORCH_DTYPE[lat]
        ZK = torch.zeros((B, Hkv, L_cap, r), dtype=zt)
        ZV = torch.zeros((B, Hkv, L_cap, r), dtype=zt)
    elif lat == "i8":
        ZK = torch.zeros((B, Hkv, L_cap, r), dtype=torch.int8)
        ZV = torch.zeros((B, Hkv, L_cap, r), dtype=torch.int8)
    elif lat == "e4m3":
        ZK = torch.zeros((B, Hkv, L_cap, r), dtype=torch.uint8)
        ZV = torch.zeros((B, Hkv, L_cap, r), dtype=torch.uint8)
    else:
        raise ValueError(lat)
    quant = lat in ("i8", "e4m3")
    SK = torch.zeros((B, Hkv, L_cap), dtype=torch.float32) if quant else None
    SV = torch.zeros((B, Hkv, L_cap), dtype=torch.float32) if quant else None

    for b in range(B):
        Lb = int(seqlens[b])
        mult = np.ones(Lb)
        if wl.outlier_frac > 0.0 and Lb > 0:
            n_out = int(math.floor(wl.outlier_frac * Lb))
            idx = rng.choice(Lb, size=n_out, replace=False)
            mult[idx] = wl.outlier_scale
        for which, Z, S in (("K", ZK, SK), ("V", ZV, SV)):
            if lat in ("f32", "bf16"):
                z = rng.standard_normal((Hkv, Lb, r)) * mult[None, :, None]
                Z[b, :, :Lb, :] = torch.from_numpy(z).to(Z.dtype)
            elif lat == "i8":
                z = rng.standard_normal((Hkv, Lb, r)) * mult[None, :, None] * (127.0 / 3.0)
                codes = np.clip(np.rint(z), -127, 127).astype(np.int8)
                Z[b, :, :Lb, :] = torch.from_numpy(codes)
                s = (3.0 / 127.0) * rng.uniform(0.8, 1.2, size=(Hkv, Lb))
                S[b, :, :Lb] = torch.from_numpy(s.astype(np.float32))
            else:
                z = rng.standard_normal((Hkv, Lb, r)) * mult[None, :, None] * (448.0 / 4.0)
                z = np.clip(z, -448.0, 448.0).astype(np.float32)
                codes = torch.from_numpy(z).to(torch.float8_e4m3fn).view(torch.uint8)
                Z[b, :, :Lb, :] = codes
                s = (4.0 / 448.0) * rng.uniform(0.8, 1.2, size=(Hkv, Lb))
                S[b, :, :Lb] = torch.from_numpy(s.astype(np.float32))

    if poison is not None:
        for b in range(B):
            Lb = int(seqlens[b])
            if Lb >= L_cap:
                continue
            for Z in (ZK, ZV):
                if lat == "f32" or lat == "bf16":
                    Z[b, :, Lb:, :] = float("nan") if poison == "nan" else 1e30
                elif lat == "i8":
                    Z[b, :, Lb:, :] = 127
                else:
                    Z[b, :, Lb:, :] = 0x7F if poison == "nan" else 0x7E  # NaN / 448
            for S in (SK, SV):
                if S is not None:
                    S[b, :, Lb:] = float("nan") if poison == "nan" else 1e30

    out.update(ZK=ZK, ZV=ZV, ZK_scale=SK, ZV_scale=SV)
    return out


def with_text_factors(wl: Workload, inputs: dict) -> dict:
    """Modality-separated factors: a copy of ``inputs`` whose BK/BV are [2][Hkv][r][d],
    the workload's own factors (the visual set) followed by a second set drawn the same
    way from another seed (the text set)."""
    rng = np.random.default_rng(np.random.PCG64(wl.seed + 1000))
    sig = sigmas(wl)
    io_t = _TORCH_DTYPE[wl.io_dtype]
    out = dict(inputs)
    for k in ("BK", "BV"):
        f = np.stack([sig[:, None] * _orthonormal_rows(rng, wl.rank, wl.d_head)
                      for _ in range(wl.n_kv_heads)])
        text = torch.from_numpy(np.ascontiguousarray(f)).to(io_t)
        out[k] = torch.stack([inputs[k], text]).contiguous()
    return out


def make_append_rows(wl: Workload, step: int = 0) -> dict:
    """New latent rows for one append: zk_new, zv_new [B][Hkv][r] in the io dtype."""
    rng = np.random.default_rng(np.random.PCG64(wl.seed * 7919 + 13 + step))
    io_t = _TORCH_DTYPE[wl.io_dtype]
    shape = (wl.batch, wl.n_kv_heads, wl.rank)
    zk = rng.standard_normal(shape)
    zv = rng.standard_normal(shape)
    return {"zk_new": torch.from_numpy(zk).to(io_t), "zv_new": torch.from_numpy(zv).to(io_t)}


def stored_bits(t: Optional[torch.Tensor]) -> Optional[np.ndarray]:
    """Raw stored representation as numpy (bf16 -> uint16 bits, e4m3 -> uint8 codes)."""
    if t is None:
        return None
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()
