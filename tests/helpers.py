"""Shared test helpers: move workload inputs to the GPU, call the C ABI through the
binding, and evaluate the oracle on the same stored inputs."""
from __future__ import annotations

import numpy as np
import torch

from oracle import lrkv_oracle as orc
from rank_kv_cache_head_b200 import lrkv
from rank_kv_cache_head_b200.workloads import stored_bits

# tolerances for decode attention against the fp64 oracle
TOL_F32_MAXABS = 1e-5
TOL_LOWP_MAXABS = 2e-2
TOL_LOWP_RELL2 = 5e-3


def dims_for(wl, inputs, num_splits=0, algo="auto", max_seqlen=None):
    L_cap = inputs["ZK"].shape[2]
    if max_seqlen is None:
        max_seqlen = int(inputs["seqlens"].max()) if inputs["seqlens"].numel() else 0
    return lrkv.make_dims(wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.d_head, wl.rank, L_cap,
                          max_seqlen, wl.io_dtype, wl.latent_dtype, num_splits, algo)


def to_device(inputs, device="cuda"):
    return {k: (None if v is None else v.to(device)) for k, v in inputs.items()}


def run_gpu(wl, inputs, num_splits=0, algo="auto", max_seqlen=None, dev=None, ws=None):
    """One lrkv_decode_attn call. Returns (out fp64 numpy, lse numpy, status, dims)."""
    dims = dims_for(wl, inputs, num_splits, algo, max_seqlen)
    dev = dev if dev is not None else to_device(inputs)
    io_t = torch.float32 if wl.io_dtype == "f32" else torch.bfloat16
    out = torch.full((wl.batch, wl.n_q_heads, wl.d_head), float("nan"), dtype=io_t,
                     device="cuda")
    lse = torch.full((wl.batch, wl.n_q_heads), float("nan"), dtype=torch.float32, device="cuda")
    ws = ws if ws is not None else lrkv.new_workspace(dims)
    lrkv.decode_attn(dims, dev["q"], dev["ZK"], dev["ZV"], dev["ZK_scale"], dev["ZV_scale"],
                     dev["BK"], dev["BV"], dev["seqlens"], out, ws, lse_out=lse)
    status = lrkv.read_status(ws)
    return out.double().cpu().numpy(), lse.cpu().numpy().astype(np.float64), status, dims


def oracle_inputs(wl, inputs):
    """Decode the stored inputs to float64 with the oracle's own decoders."""
    io = wl.io_dtype
    lat = wl.latent_dtype
    dec = lambda t, dt: None if t is None else orc.decode_stored(stored_bits(t), dt)
    return dict(q=dec(inputs["q"], io), ZK=dec(inputs["ZK"], lat), ZV=dec(inputs["ZV"], lat),
                BK=dec(inputs["BK"], io), BV=dec(inputs["BV"], io),
                ZK_scale=None if inputs["ZK_scale"] is None else inputs["ZK_scale"].numpy().astype(np.float64),
                ZV_scale=None if inputs["ZV_scale"] is None else inputs["ZV_scale"].numpy().astype(np.float64),
                seqlens=inputs["seqlens"].numpy())


def run_oracle(wl, inputs, pairs=None):
    o = oracle_inputs(wl, inputs)
    return orc.decode_attention(o["q"], o["ZK"], o["ZV"], o["BK"], o["BV"], o["seqlens"],
                                o["ZK_scale"], o["ZV_scale"], pairs=pairs)


def compare(wl, got, ref, got_lse=None, ref_lse=None, rows=None, lse_bound=None):
    """Assert the tolerance for the workload's io dtype. ``rows`` selects (b, h)."""
    if rows is not None:
        idx = tuple(np.array(rows).T)
        got, ref = got[idx], ref[idx]
        if got_lse is not None:
            got_lse, ref_lse = got_lse[idx], ref_lse[idx]
        if lse_bound is not None:
            lse_bound = lse_bound[idx]
    assert np.all(np.isfinite(got)), "non-finite output"
    err = np.abs(got - ref)
    max_abs = float(err.max()) if err.size else 0.0
    nrm = float(np.linalg.norm(ref))
    rel_l2 = float(np.linalg.norm(got - ref) / nrm) if nrm > 0 else float(np.linalg.norm(got))
    if wl.io_dtype == "f32":
        assert max_abs <= TOL_F32_MAXABS, f"max-abs {max_abs:.3e} > {TOL_F32_MAXABS}"
    else:
        assert max_abs <= TOL_LOWP_MAXABS, f"max-abs {max_abs:.3e} > {TOL_LOWP_MAXABS}"
        assert rel_l2 <= TOL_LOWP_RELL2, f"rel-L2 {rel_l2:.3e} > {TOL_LOWP_RELL2}"
    if got_lse is not None:
        both_inf = np.isneginf(got_lse) & np.isneginf(ref_lse)
        d = np.abs(np.where(both_inf, 0.0, got_lse - ref_lse))
        assert np.all(np.isfinite(d)), "lse mismatch in finiteness"
        tol = 1e-5 if wl.io_dtype == "f32" else 1e-3
        if lse_bound is not None:
            tol = tol + lse_bound
        assert np.all(d <= tol), f"lse err {float(np.max(d - tol)):.3e} above its bound"
    return max_abs, rel_l2


def lse_rounding_bound(wl, inputs, rows=None):
    """Per-(b, h) bound on the LSE error of a 16-bit tensor-core score path: the
    rebuilt keys are rounded to f16 (relative error <= 2^-11 per element) before
    the q K^T contraction, so every score moves by at most
    2^-11 * sum_c |q_c K_tc| / sqrt(d), and the LSE by at most the largest such move.
    Doubled for the fp32 accumulation and the q conversion. Zero for fp32 I/O."""
    if wl.io_dtype == "f32":
        return None
    o = oracle_inputs(wl, inputs)
    B, Hq, d = o["q"].shape
    G = Hq // o["ZK"].shape[1]
    bound = np.zeros((B, Hq))
    for b in range(B):
        L = int(o["seqlens"][b])
        if L <= 0:
            continue
        for h in range(Hq):
            if rows is not None and (b, h) not in rows:
                continue
            g = h // G
            Z = o["ZK"][b, g, :L]
            if o["ZK_scale"] is not None:
                Z = Z * o["ZK_scale"][b, g, :L, None]
            K = Z @ o["BK"][g]
            bound[b, h] = 2.0 * 2.0 ** -11 * float(np.max(np.abs(K) @ np.abs(o["q"][b, h]))) / np.sqrt(d)
    return bound
