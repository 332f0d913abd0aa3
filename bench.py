#!/usr/bin/env python
"""Decode-step benchmark for low-rank (per-head SVD-factored) KV-cache attention.

One step = one decode step of one layer for every batch row: lrkv_append writes the
new token's latent row per (batch row, KV head), then lrkv_decode_attn runs the
split-KV kernel (rebuild K = Z_K B_K, V = Z_V B_V on chip, scores, online softmax,
P V) and the log-sum-exp merge. Inputs are seeded synthetic workloads (see
rank_kv_cache_head_b200/workloads.py) resident in HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--algo auto|simt|tcgen05] [--impl ours|reference]

Timing: the K steps are captured into CUDA graphs and replayed; the timed region is
bracketed by a barrier and torch.cuda.synchronize on both sides and measured with
CUDA events on the launching stream, max over ranks. The cache is rotated among
enough copies that the bytes touched between two uses of a copy exceed 3x the L2
size, and every copy's seqlens is restored on a parallel graph branch after its
step, so each step attends exactly the workload's lengths. Events recorded in the
graph around every split-kernel launch give the dominant kernel's duration.
With --gpus N > 1 (torchrun), every rank runs its own batch (weak scaling, no
collective on the data path) and rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import glob
import json
import math
import os
import statistics
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from rank_kv_cache_head_b200 import lrkv  # noqa: E402
from rank_kv_cache_head_b200.metrics import (ClockSampler, max_over_ranks,  # noqa: E402
                                             step_bytes, sum_over_ranks)
from rank_kv_cache_head_b200.workloads import (WORKLOADS, make_append_rows,  # noqa: E402
                                               make_inputs, seqlens_for, with_text_factors)

METRIC = "low-rank decode attention: latent GB/s, tokens/s/GPU, % of HBM roofline"
UNIT = "GB/s"
DEFAULT_WORKLOAD = "vlm7b-bf16"
L2_BYTES = 126 * 1024 ** 2
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--algo", default="auto", choices=["auto", "simt", "tcgen05"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="CPU time budget of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=100)
    ap.add_argument("--projection-dmodel", type=int, default=4096,
                    help="also time lrkv_project_append with this hidden size (0: skip)")
    ap.add_argument("--adaptive-rlow", type=int, default=0, metavar="R",
                    help="also time the attention-aware partial decompression with tokens "
                         "below the importance threshold rebuilt at rank R (0: skip)")
    ap.add_argument("--shared-rank", type=int, default=0, metavar="R",
                    help="also time decode attention over a cross-head shared latent of rank "
                         "R on this workload's shape (0: skip)")
    ap.add_argument("--n-visual", type=int, default=0, metavar="P",
                    help="modality-separated factors: positions < P use a visual factor "
                         "set, the rest a text set (0: one set, the default)")
    ap.add_argument("--profile", type=int, default=0, metavar="N",
                    help="no timing: run N eager decode-attention calls on one cache copy "
                         "and exit (a short, fixed launch sequence for ncu captures)")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def dist_init():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world <= 1:
        return 0, 1, 0
    import torch.distributed as dist
    rank = int(os.environ["RANK"])
    local = int(os.environ.get("LOCAL_RANK", rank))
    if torch.cuda.is_available():
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
    return rank, world, local


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def kernel_source_hash() -> str:
    """Hash of the split kernel's sources (the kernel file and the headers it includes):
    DRAM counters taken on other sources do not describe it."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "rank_kv_cache_head_b200", "csrc")
    for name in ("lrkv_tc.cu", "lrkv_sm100.cuh", "lrkv_tmap.h", "lrkv_internal.h"):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    inc = os.path.join(ROOT, "include", "lrkv.h")
    with open(inc, "rb") as f:
        h.update(b"lrkv.h" + f.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str, algo: str):
    """DRAM bytes per split-kernel launch from the committed ncu summary, if it was
    taken on the current kernel sources (else None)."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(p) as f:
            j = json.load(f)
    except (OSError, ValueError):
        return None
    e = j.get(f"{workload}/{algo}")
    if not e or e.get("kernel_source_hash") != kernel_source_hash():
        return None
    return e.get("dram_bytes_per_launch")


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


# ---------------------------------------------------------------------------------------
# CPU oracle timing (the reference arm and the cpu_baseline field)
# ---------------------------------------------------------------------------------------


def oracle_sample(wl, inputs, budget_s: float, max_units=None, rng_seed=0, n_visual=0):
    """Time the fp64 oracle on whole (batch row, KV head) units in a seeded random
    order until ``budget_s`` seconds of work are done. Returns (seconds per unit,
    units timed, latent bytes timed, seconds)."""
    from oracle import lrkv_oracle as orc
    from rank_kv_cache_head_b200.workloads import stored_bits
    io, lat = wl.io_dtype, wl.latent_dtype
    q = orc.decode_stored(stored_bits(inputs["q"]), io)
    BK = orc.decode_stored(stored_bits(inputs["BK"]), io)
    BV = orc.decode_stored(stored_bits(inputs["BV"]), io)
    seq = inputs["seqlens"].numpy()
    units = [(b, g) for b in range(wl.batch) for g in range(wl.n_kv_heads)]
    order = np.random.default_rng(rng_seed).permutation(len(units))
    G = wl.group
    spent, n, lat_bytes = 0.0, 0, 0
    per_tok = 2 * wl.rank * {"f32": 4, "bf16": 2, "i8": 1, "e4m3": 1}[lat] + \
        (8 if lat in ("i8", "e4m3") else 0)
    for i in order:
        b, g = units[i]
        Lb = int(seq[b])
        # decode this unit's stored rows (part of the oracle's work)
        t0 = time.perf_counter()
        ZK = orc.decode_stored(stored_bits(inputs["ZK"][b:b + 1, g:g + 1, :Lb]), lat)
        ZV = orc.decode_stored(stored_bits(inputs["ZV"][b:b + 1, g:g + 1, :Lb]), lat)
        SK = SV = None
        if inputs["ZK_scale"] is not None:
            SK = inputs["ZK_scale"][b:b + 1, g:g + 1, :Lb].numpy().astype(np.float64)
            SV = inputs["ZV_scale"][b:b + 1, g:g + 1, :Lb].numpy().astype(np.float64)
        if n_visual:     # factors [2][Hkv][r][d]: both sets of this head
            orc.decode_attention(q[b:b + 1, g * G:(g + 1) * G], ZK, ZV, BK[:, g:g + 1],
                                 BV[:, g:g + 1], np.array([Lb]), SK, SV, n_visual=n_visual)
        else:
            orc.decode_attention(q[b:b + 1, g * G:(g + 1) * G], ZK, ZV, BK[g:g + 1], BV[g:g + 1],
                                 np.array([Lb]), SK, SV)
        spent += time.perf_counter() - t0
        n += 1
        lat_bytes += Lb * per_tok
        if spent >= budget_s or (max_units is not None and n >= max_units):
            break
    return spent / max(n, 1), n, lat_bytes, spent


def run_reference(args, rank):
    """The oracle as it stands, timed on the host cores: each step is a bounded sample
    (one (batch row, KV head) unit, all its query heads) of the workload."""
    if rank != 0:
        return
    wl = WORKLOADS[args.workload]
    target = seqlens_for(wl)
    inputs = make_inputs(wl, capacity=int(target.max()), seqlens=target)
    for _ in range(args.warmup):
        oracle_sample(wl, inputs, 0.0, max_units=1, rng_seed=1)
    times, byts = [], 0
    for k in range(args.steps):
        per_unit, n, lb, spent = oracle_sample(wl, inputs, 0.0, max_units=1, rng_seed=100 + k)
        times.append(spent)
        byts += lb
    total = sum(times)
    units_per_step = wl.batch * wl.n_kv_heads
    sec_per_full_step = statistics.mean(times) * units_per_step
    value = byts / total / 1e9
    cores = blas_threads()
    sample = (f"{args.steps} steps, each one (batch row, KV head) unit of {args.workload} "
              f"({wl.group} query heads), fp64 numpy oracle, {cores} BLAS threads")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": statistics.mean(times) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(wl, target, None, "oracle"),
        "tokens_per_s_per_gpu": wl.batch / sec_per_full_step,
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(wl, target, plan, algo):
    cfg = {"workload": wl.name, "batch": wl.batch, "n_q_heads": wl.n_q_heads,
           "n_kv_heads": wl.n_kv_heads, "d_head": wl.d_head, "rank": wl.rank,
           "seq_len": int(target.max()) if wl.ragged_min is None else
           f"ragged U[{wl.ragged_min},{wl.seq_len}] (mean {float(np.mean(target)):.1f})",
           "io_dtype": wl.io_dtype, "latent_dtype": wl.latent_dtype, "kernel": algo}
    if plan is not None:
        cfg["plan"] = plan
    return cfg


# ---------------------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------------------


def event_ms(a, b) -> float:
    """Elapsed ms between two events the library recorded as graph nodes (torch's own
    elapsed_time only accepts events recorded through torch)."""
    from cuda.bindings import runtime as rt
    err, ms = rt.cudaEventElapsedTime(a.cuda_event, b.cuda_event)
    if int(err) != 0:
        raise RuntimeError(f"cudaEventElapsedTime failed: {err}")
    return float(ms)


def largest_divisor_at_most(k: int, cap: int) -> int:
    for g in range(min(k, cap), 0, -1):
        if k % g == 0:
            return g
    return 1


def measure_projection(wl, dev, d_model: int):
    """Time lrkv_project_append (the fused latent projection + append that produces each
    step's new latent rows) on this workload's cache shape, with a d_model-wide hidden
    state. The factors A_K, A_V are rotated over >= 3x L2 of copies; every call appends
    at a fresh slot. Returns a dict for the JSON line."""
    g = torch.Generator(device="cpu").manual_seed(wl.seed + 99)
    io_t = torch.float32 if wl.io_dtype == "f32" else torch.bfloat16
    H, r, B = wl.n_kv_heads, wl.rank, wl.batch
    a_bytes = 2 * H * d_model * r * (4 if wl.io_dtype == "f32" else 2)
    n_a = max(2, min(48, math.ceil(3 * L2_BYTES / a_bytes)))
    A = [(torch.randn(H, d_model, r, generator=g) / math.sqrt(d_model)).to(io_t).to(dev)
         for _ in range(2 * n_a)]
    x = torch.randn(B, d_model, generator=g).to(io_t).to(dev)
    per_graph, replays, warm = 40, 3, 5
    cap = warm + per_graph * (replays + 1) + 16
    lat_t = {"f32": torch.float32, "bf16": torch.bfloat16, "i8": torch.int8,
             "e4m3": torch.uint8}[wl.latent_dtype]
    ZK = torch.zeros(B, H, cap, r, dtype=lat_t, device=dev)
    ZV = torch.zeros_like(ZK)
    quant = wl.latent_dtype in ("i8", "e4m3")
    SK = torch.ones(B, H, cap, dtype=torch.float32, device=dev) if quant else None
    SV = torch.ones_like(SK) if quant else None
    seq = torch.zeros(B, dtype=torch.int32, device=dev)
    dims = lrkv.make_dims(B, wl.n_q_heads, H, wl.d_head, r, cap, cap, wl.io_dtype,
                          wl.latent_dtype)
    ws = torch.zeros(max(lrkv.workspace_bytes(dims), 1 << 20), dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(device=dev)
    call = lambda i: lrkv.project_append(dims, x, A[2 * (i % n_a)], A[2 * (i % n_a) + 1], ZK, ZV,
                                         SK, SV, seq, ws, stream=stream)
    with torch.cuda.stream(stream):
        for i in range(warm):
            call(i)
        stream.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            for i in range(per_graph):
                call(i)
        graph.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(replays):
            graph.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    n = per_graph * replays
    us = e0.elapsed_time(e1) * 1e3 / n
    st = lrkv.read_status(ws)
    if st:
        raise RuntimeError(f"device status {st} after the projection timing")
    lat_bytes = {"f32": 4, "bf16": 2, "i8": 1, "e4m3": 1}[wl.latent_dtype]
    moved = a_bytes + x.numel() * x.element_size() + 2 * B * H * r * lat_bytes + (
        2 * B * H * 4 if quant else 0)
    peak, kind = peaks()
    return {"d_model": d_model, "us_per_call": us, "bytes_per_call": moved,
            "achieved_GBs": moved / (us * 1e-6) / 1e9, "peak_GBs": peak, "peak_kind": kind,
            "frac": moved / (us * 1e-6) / 1e9 / peak, "launches": "CUDA graph of 40 calls",
            "factors": f"rotated over {n_a} copies ({n_a * a_bytes / 1e6:.0f} MB)"}


def measure_adaptive(wl, dev, r_low: int, tau: float = 0.5, beta: float = 0.9):
    """Time lrkv_decode_attn_adaptive (attention-aware partial decompression, CUDA-core
    kernel) on this workload beside the plain CUDA-core decode of the same cache: about
    half of the tokens (importance drawn uniform in [0, 1], tau 0.5) are rebuilt at rank
    r_low. Each timed call also updates the importance. Returns a dict for the JSON line."""
    target = seqlens_for(wl)
    cap = ((int(target.max()) + 7) // 8) * 8
    x = make_inputs(wl, capacity=cap, seqlens=target)
    d = {k: (None if v is None else v.to(dev)) for k, v in x.items()}
    dims = lrkv.make_dims(wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.d_head, wl.rank, cap,
                          int(target.max()), wl.io_dtype, wl.latent_dtype, 0, "simt")
    g = torch.Generator(device="cpu").manual_seed(wl.seed + 77)
    imp = torch.rand(wl.batch, wl.n_kv_heads, cap, generator=g).to(dev)
    low_frac = float((imp.cpu()[..., :int(target.max())] < tau).float().mean())
    scores = torch.empty(wl.batch, wl.n_q_heads, cap, dtype=torch.float32, device=dev)
    out = torch.empty_like(d["q"])
    lse = torch.empty(wl.batch, wl.n_q_heads, dtype=torch.float32, device=dev)
    ws = lrkv.new_workspace(dims, device=dev)
    stream = torch.cuda.Stream(device=dev)
    adaptive = lambda: lrkv.decode_attn_adaptive(dims, d["q"], d["ZK"], d["ZV"], d["ZK_scale"],
                                                 d["ZV_scale"], d["BK"], d["BV"], d["seqlens"], imp,
                                                 tau, r_low, beta, scores, out, lse, ws, stream=stream)
    plain = lambda: lrkv.decode_attn(dims, d["q"], d["ZK"], d["ZV"], d["ZK_scale"], d["ZV_scale"],
                                     d["BK"], d["BV"], d["seqlens"], out, ws, lse_out=lse,
                                     stream=stream)
    per_graph, replays = 10, 3

    def time_it(fn):
        with torch.cuda.stream(stream):
            for _ in range(3):
                fn()
            stream.synchronize()
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=stream):
                for _ in range(per_graph):
                    fn()
            graph.replay()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(replays):
                graph.replay()
            e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) * 1e3 / (per_graph * replays)

    us_plain = time_it(plain)
    us_adapt = time_it(adaptive)
    st = lrkv.read_status(ws)
    if st:
        raise RuntimeError(f"device status {st} after the adaptive timing")
    sb = step_bytes(wl, target)
    lat = sb["latent"] + sb["scales"]
    peak, kind = peaks()
    return {"kernel": "CUDA-core split (simt) + merge + attention-mass moving average",
            "r_low": r_low, "rank": wl.rank, "tau": tau, "beta": beta,
            "low_rank_token_fraction": low_frac,
            "reconstruction_flops_fraction": low_frac * r_low / wl.rank + (1 - low_frac),
            "us_per_call": us_adapt, "simt_plain_us_per_call": us_plain,
            "latent_GBs": lat / (us_adapt * 1e-6) / 1e9, "peak_GBs": peak, "peak_kind": kind,
            "frac": lat / (us_adapt * 1e-6) / 1e9 / peak,
            "launches": f"CUDA graph of {per_graph} calls, one cache copy"}


def measure_shared(wl, dev, R: int):
    """Time lrkv_decode_attn_shared (cross-head shared latent, CUDA-core kernel) on this
    workload's batch, heads and lengths with one rank-R latent row per token for every
    KV head (bf16 latents and decompression matrices, seeded). Returns a dict."""
    target = seqlens_for(wl)
    cap = ((int(target.max()) + 7) // 8) * 8
    g = torch.Generator(device="cpu").manual_seed(wl.seed + 55)
    io_t = torch.float32 if wl.io_dtype == "f32" else torch.bfloat16
    B, Hq, Hkv, d = wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.d_head
    q = torch.randn(B, Hq, d, generator=g).to(io_t).to(dev)
    ZK = torch.randn(B, cap, R, generator=g).to(io_t).to(dev)
    ZV = torch.randn(B, cap, R, generator=g).to(io_t).to(dev)
    DK = (torch.randn(R, Hkv * d, generator=g) / math.sqrt(R)).to(io_t).to(dev)
    DV = (torch.randn(R, Hkv * d, generator=g) / math.sqrt(R)).to(io_t).to(dev)
    seq = torch.from_numpy(target.astype(np.int32)).to(dev)
    dims = lrkv.make_dims(B, Hq, Hkv, d, R, cap, int(target.max()), wl.io_dtype, wl.io_dtype, 0,
                          "simt")
    out = torch.empty_like(q)
    ws = lrkv.new_workspace(dims, device=dev)
    stream = torch.cuda.Stream(device=dev)
    per_graph, replays = 10, 3
    with torch.cuda.stream(stream):
        call = lambda: lrkv.decode_attn_shared(dims, q, ZK, ZV, None, None, DK, DV, seq, out, ws,
                                               stream=stream)
        for _ in range(3):
            call()
        stream.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            for _ in range(per_graph):
                call()
        graph.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(replays):
            graph.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / (per_graph * replays)
    st = lrkv.read_status(ws)
    if st:
        raise RuntimeError(f"device status {st} after the shared-latent timing")
    lat = int(target.sum()) * 2 * R * ZK.element_size()
    peak, kind = peaks()
    return {"kernel": "CUDA-core split (simt, shared-latent layout) + merge", "rank": R,
            "latent_bytes_per_token": 2 * R * ZK.element_size(),
            "per_head_equivalent_bytes_per_token": 2 * wl.rank * Hkv * ZK.element_size(),
            "us_per_call": us, "latent_GBs": lat / (us * 1e-6) / 1e9, "peak_GBs": peak,
            "peak_kind": kind, "frac": lat / (us * 1e-6) / 1e9 / peak,
            "launches": f"CUDA graph of {per_graph} calls"}


def run_ours(args, rank, world, local):
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    wl = WORKLOADS[args.workload]
    target = seqlens_for(wl)                         # attended lengths (after append)
    Lmax = int(target.max())
    capacity = ((Lmax + args.e2e_steps + 16 + 7) // 8) * 8
    inputs = make_inputs(wl, capacity=capacity, seqlens=target)
    if args.n_visual:
        inputs = with_text_factors(wl, inputs)
    sb = step_bytes(wl, target, factor_sets=2 if args.n_visual else 1)
    per_copy = sb["latent"] + sb["scales"]
    n_copies = max(2, math.ceil(3 * L2_BYTES / max(per_copy, 1)))
    n_copies = min(n_copies, 64)

    dims = lrkv.make_dims(wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.d_head, wl.rank, capacity,
                          Lmax, wl.io_dtype, wl.latent_dtype, 0, args.algo, n_visual=args.n_visual)
    plan = lrkv.plan(dims)
    q = inputs["q"].to(dev)
    BK, BV = inputs["BK"].to(dev), inputs["BV"].to(dev)
    io_t = q.dtype
    out = torch.empty_like(q)
    ws = lrkv.new_workspace(dims, device=dev)
    seq0 = torch.from_numpy((target - 1).astype(np.int32)).to(dev)
    copies = []
    for c in range(n_copies):
        rows = make_append_rows(wl, step=c)
        cp = {"ZK": inputs["ZK"].to(dev), "ZV": inputs["ZV"].to(dev),
              "SK": None if inputs["ZK_scale"] is None else inputs["ZK_scale"].to(dev),
              "SV": None if inputs["ZV_scale"] is None else inputs["ZV_scale"].to(dev),
              "seq": seq0.clone(), "zk": rows["zk_new"].to(dev), "zv": rows["zv_new"].to(dev)}
        cp["step"] = lrkv.PreparedStep(dims, q, cp["ZK"], cp["ZV"], cp["SK"], cp["SV"], BK, BV,
                                       cp["seq"], out, ws, cp["zk"], cp["zv"])
        copies.append(cp)
    torch.cuda.synchronize()

    s_main = torch.cuda.Stream(device=dev)
    s_side = torch.cuda.Stream(device=dev)
    # one eager step first: one-time launch set-up never happens inside a capture
    with torch.cuda.stream(s_main):
        copies[0]["step"](s_main.cuda_stream)
        copies[0]["seq"].copy_(seq0)
    torch.cuda.synchronize()
    if lrkv.read_status(ws):
        raise RuntimeError("device status after the first eager step")
    G = largest_divisor_at_most(args.steps, 64)
    ev_b = [torch.cuda.Event(enable_timing=True) for _ in range(G)]
    ev_e = [torch.cuda.Event(enable_timing=True) for _ in range(G)]
    for ev in ev_b + ev_e:     # torch creates the underlying CUDA event on first record
        ev.record(s_main)
    torch.cuda.synchronize()

    def capture(nsteps, timed):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s_main):
            cur = torch.cuda.current_stream()
            handle = cur.cuda_stream
            pending = {}
            for k in range(nsteps):
                c = k % n_copies
                if c in pending:
                    cur.wait_event(pending.pop(c))
                if timed:
                    copies[c]["step"](handle, ev_b[k].cuda_event, ev_e[k].cuda_event)
                else:
                    copies[c]["step"](handle)
                done = torch.cuda.Event()
                done.record(cur)
                s_side.wait_event(done)
                with torch.cuda.stream(s_side):
                    copies[c]["seq"].copy_(seq0, non_blocking=True)
                    rest = torch.cuda.Event()
                    rest.record(s_side)
                pending[c] = rest
            for e in pending.values():
                cur.wait_event(e)
        return g

    props = torch.cuda.get_device_properties(dev)
    gpu_id = f"GPU-{props.uuid}" if getattr(props, "uuid", None) else str(local)
    sampler = ClockSampler(gpu_id).start()
    graph = capture(G, timed=True)
    warm_reps = max(1, math.ceil(args.warmup / G))
    with torch.cuda.stream(s_main):
        for _ in range(warm_reps):
            graph.replay()
    torch.cuda.synchronize()
    status = lrkv.read_status(ws)
    if status:
        raise RuntimeError(f"device status {status} after warm-up")

    reps = args.steps // G
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    with torch.cuda.stream(s_main):
        start.record()
        for _ in range(reps):
            graph.replay()
        end.record()
    torch.cuda.synchronize()
    t1 = time.perf_counter()
    barrier()
    ms = start.elapsed_time(end)
    split_ms = [event_ms(ev_b[k], ev_e[k]) for k in range(G)]  # last replay's launches
    status = lrkv.read_status(ws)
    if status:
        raise RuntimeError(f"device status {status} after the timed region")
    ms_max = max_over_ranks(ms, dev)
    sampler.stop()
    clocks = sampler.summary(t0, t1)

    # ---- end to end through the public host-buffer entry point --------------------------
    q_h = inputs["q"].pin_memory()
    rows0 = make_append_rows(wl, step=0)
    zk_h, zv_h = rows0["zk_new"].pin_memory(), rows0["zv_new"].pin_memory()
    out_h = torch.empty_like(inputs["q"]).pin_memory()
    q_d, o_d = torch.empty_like(q), torch.empty_like(q)
    zk_d, zv_d = torch.empty_like(copies[0]["zk"]), torch.empty_like(copies[0]["zv"])
    for cp in copies:
        cp["seq"].copy_(seq0)
    ke = max(1, args.e2e_steps)
    # the end-to-end steps keep appending, so their planning hint covers the growth
    dims_e2e = lrkv.make_dims(wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.d_head, wl.rank,
                              capacity, min(capacity, Lmax + ke // n_copies + 1), wl.io_dtype,
                              wl.latent_dtype, 0, args.algo, n_visual=args.n_visual)
    ws_e2e = lrkv.new_workspace(dims_e2e, device=dev)
    uses = [0] * n_copies
    e2e_lat = 0
    for k in range(ke):
        c = k % n_copies
        e2e_lat += step_bytes(wl, target + uses[c])["latent"] + step_bytes(wl, target + uses[c])["scales"]
        uses[c] += 1
    for cp in copies:
        cp["seq"].copy_(seq0)
    torch.cuda.synchronize()
    es, ee = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with torch.cuda.stream(s_main):
        es.record()
        for k in range(ke):
            cp = copies[k % n_copies]
            lrkv.decode_step_host(dims_e2e, q_h, zk_h, zv_h, out_h, q_d, zk_d, zv_d, o_d,
                                  cp["ZK"], cp["ZV"], cp["SK"], cp["SV"], BK, BV, cp["seq"],
                                  ws_e2e, stream=s_main)
            s_main.synchronize()          # the step's result is read on the host
            _ = out_h[0, 0, 0].item()
        ee.record()
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(es.elapsed_time(ee), dev)
    st_e2e = lrkv.read_status(ws_e2e)
    if st_e2e:
        raise RuntimeError(f"device status {st_e2e} after the end-to-end loop")

    # ---- numbers -------------------------------------------------------------------------
    peak, peak_kind = peaks()
    lat_step = sb["latent"] + sb["scales"]
    total_lat = sum_over_ranks(lat_step * args.steps, dev)
    value = total_lat / (ms_max * 1e-3) / 1e9
    split_mean_ms = statistics.mean(split_ms)
    achieved = sb["split_kernel"] / (split_mean_ms * 1e-3) / 1e9
    traffic = profiled_traffic(args.workload, plan["algo"])
    if plan.get("device_chunk"):
        # the split size the kernel picked from the lengths (header word 4)
        plan["chunk_chosen"] = int(ws[16:20].view(torch.int32).item())
    e2e_value = sum_over_ranks(e2e_lat, dev) / (e2e_ms * 1e-3) / 1e9
    io_bytes = 4 if wl.io_dtype == "f32" else 2
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": warm_reps * G, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": {"bf16": "bf16", "f32": "f32"}[wl.io_dtype] + (
            "" if wl.latent_dtype in ("bf16", "f32") else f"+{wl.latent_dtype}-latents"),
        "data": "synthetic (seeded; shapes and distributions of the workload definition)",
        "config": dict(workload_config(wl, target, plan, plan["algo"]),
                       **({"n_visual": args.n_visual,
                           "factors": "modality-separated (visual set below n_visual, text set after)"}
                          if args.n_visual else {}),
                       parallelism=f"dp{world} (independent batches per GPU)",
                       l2=f"cache rotated over {n_copies} copies ({n_copies * per_copy / 1e6:.0f} MB "
                          f">= 3x L2) between uses"),
        "tokens_per_s_per_gpu": wl.batch * args.steps / (ms_max * 1e-3),
        "hbm_roofline_frac": sb["total"] * args.steps / (ms_max * 1e-3) / 1e9 / peak,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "kernel": f"split ({plan['algo']})", "peak_kind": peak_kind,
                     "split_us_mean": split_mean_ms * 1e3,
                     "bytes_per_launch": sb["split_kernel"]},
        "e2e": {"value": e2e_value, "unit": UNIT,
                "h2d_bytes_per_step": q.numel() * io_bytes + 2 * zk_d.numel() * io_bytes,
                "d2h_bytes_per_step": q.numel() * io_bytes, "steps": ke,
                "ms_per_step": e2e_ms / ke},
        "gpu_launches": 3 * args.steps,
        "clocks": clocks,
        "cpu_baseline": None,
    }
    if args.projection_dmodel > 0:
        line["project_append"] = measure_projection(wl, dev, args.projection_dmodel)
    if rank == 0 and args.adaptive_rlow > 0:
        line["adaptive"] = measure_adaptive(wl, dev, args.adaptive_rlow)
    if rank == 0 and args.shared_rank > 0:
        line["shared_latent"] = measure_shared(wl, dev, args.shared_rank)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        per_unit, n, lb, spent = oracle_sample(wl, inputs, args.cpu_seconds, n_visual=args.n_visual)
        cores = blas_threads()
        cpu_val = lb / spent / 1e9
        line["cpu_baseline"] = {
            "value": cpu_val, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{n} of {wl.batch * wl.n_kv_heads} (batch row, KV head) units, "
                      f"{spent:.1f} s, fp64 numpy oracle",
            "tokens_per_s": wl.batch / (per_unit * wl.batch * wl.n_kv_heads)}
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_profile(args):
    """N eager lrkv_decode_attn calls on one copy of the workload (for profilers)."""
    wl = WORKLOADS[args.workload]
    target = seqlens_for(wl)
    Lmax = int(target.max())
    capacity = ((Lmax + 7) // 8) * 8
    inputs = make_inputs(wl, capacity=capacity, seqlens=target)
    dims = lrkv.make_dims(wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.d_head, wl.rank, capacity,
                          Lmax, wl.io_dtype, wl.latent_dtype, 0, args.algo)
    dev = {k: (None if v is None else v.cuda()) for k, v in inputs.items()}
    out = torch.empty_like(dev["q"])
    ws = lrkv.new_workspace(dims)
    for _ in range(args.profile):
        lrkv.decode_attn(dims, dev["q"], dev["ZK"], dev["ZV"], dev["ZK_scale"], dev["ZV_scale"],
                         dev["BK"], dev["BV"], dev["seqlens"], out, ws)
    torch.cuda.synchronize()
    st = lrkv.read_status(ws)
    print(json.dumps({"profile_calls": args.profile, "workload": wl.name, "status": st,
                      "plan": lrkv.plan(dims)}))
    if st:
        raise SystemExit(1)


def main():
    args = parse()
    if args.profile:
        run_profile(args)
        return
    rank, world, local = dist_init()
    try:
        if args.impl == "reference":
            run_reference(args, rank)
        else:
            if not torch.cuda.is_available():
                raise SystemExit("bench.py needs a CUDA GPU for --impl ours")
            run_ours(args, rank, world, local)
    finally:
        import torch.distributed as dist
        if dist.is_available() and dist.is_initialized():
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
