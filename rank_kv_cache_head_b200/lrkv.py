"""Python binding of liblrkv.so (include/lrkv.h): argument marshalling only.

Every function here forwards torch tensors' device pointers and the current CUDA
stream to the C ABI of the same name; all arithmetic runs in the library's CUDA
kernels. There is no fallback: if liblrkv.so is missing or a call fails, an
exception is raised. Build the library with ``python -m rank_kv_cache_head_b200.build``.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblrkv.so")

F32, BF16, I8, E4M3 = 0, 1, 2, 3
DTYPE_CODE = {"f32": F32, "bf16": BF16, "i8": I8, "e4m3": E4M3}
ALGO_AUTO, ALGO_SIMT, ALGO_TCGEN05 = 0, 1, 2
ALGO_CODE = {"auto": ALGO_AUTO, "simt": ALGO_SIMT, "tcgen05": ALGO_TCGEN05}

STATUS_SEQLEN_RANGE = 1
STATUS_SEQLEN_HINT = 2
STATUS_APPEND_FULL = 4
STATUS_TIMEOUT = 8

_TORCH_OF = {F32: torch.float32, BF16: torch.bfloat16, I8: torch.int8, E4M3: torch.uint8}
_LATENT_TORCH_OK = {F32: (torch.float32,), BF16: (torch.bfloat16,), I8: (torch.int8,),
                    E4M3: (torch.uint8, torch.float8_e4m3fn)}


class LrkvError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {code} ({strerror(code)})")
        self.code = code


class Dims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "batch", "n_q_heads", "n_kv_heads", "d_head", "rank", "max_seq", "max_seqlen",
        "io_dtype", "latent_dtype", "num_splits", "algo", "n_visual")]

    def __repr__(self):
        return "Dims(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_) + ")"


class PlanInfo(ctypes.Structure):
    _fields_ = [("algo", ctypes.c_int32), ("num_splits", ctypes.c_int32),
                ("chunk", ctypes.c_int32), ("grid", ctypes.c_int32),
                ("smem_bytes", ctypes.c_int32), ("full_chunk", ctypes.c_int32),
                ("device_chunk", ctypes.c_int32), ("reserved", ctypes.c_int32)]


_lib = None
_vp = ctypes.c_void_p


def lib() -> ctypes.CDLL:
    """Load liblrkv.so once (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m rank_kv_cache_head_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        dp = ctypes.POINTER(Dims)
        L.lrkv_version.restype = ctypes.c_int
        L.lrkv_strerror.restype = ctypes.c_char_p
        L.lrkv_strerror.argtypes = [ctypes.c_int]
        L.lrkv_plan.argtypes = [dp, ctypes.POINTER(PlanInfo)]
        L.lrkv_workspace_bytes.restype = ctypes.c_size_t
        L.lrkv_workspace_bytes.argtypes = [dp]
        L.lrkv_workspace_init.argtypes = [_vp, ctypes.c_size_t, _vp]
        L.lrkv_decode_attn.argtypes = [dp] + [_vp] * 11 + [ctypes.c_size_t, _vp]
        L.lrkv_decode_attn_timed.argtypes = [dp] + [_vp] * 11 + [ctypes.c_size_t, _vp, _vp, _vp]
        L.lrkv_append.argtypes = [dp] + [_vp] * 8 + [ctypes.c_size_t, _vp]
        L.lrkv_decode_attn_noalloc.argtypes = [dp] + [_vp] * 12
        L.lrkv_decode_step_host.argtypes = [dp] + [_vp] * 16 + [ctypes.c_size_t, _vp]
        L.lrkv_read_status.argtypes = [_vp, _vp, ctypes.POINTER(ctypes.c_uint32)]
        L.lrkv_debug_stall_next_launch.argtypes = [ctypes.c_int32]
        L.lrkv_project_append.argtypes = [dp, ctypes.c_int32] + [_vp] * 9 + [ctypes.c_size_t, _vp]
        L.lrkv_decode_attn_shared.argtypes = [dp] + [_vp] * 11 + [ctypes.c_size_t, _vp]
        L.lrkv_decode_attn_adaptive.argtypes = ([dp] + [_vp] * 9 + [ctypes.c_float, ctypes.c_int32,
                                                 ctypes.c_float] + [_vp] * 4 +
                                                [ctypes.c_size_t, _vp])
        _lib = L
    return _lib


def version() -> int:
    return lib().lrkv_version()


def strerror(code: int) -> str:
    return lib().lrkv_strerror(code).decode()


def make_dims(batch, n_q_heads, n_kv_heads, d_head, rank, max_seq, max_seqlen,
              io_dtype="bf16", latent_dtype="bf16", num_splits=0, algo="auto",
              n_visual=0) -> Dims:
    """n_visual > 0: modality-separated factors, BK/BV [2][Hkv][r][d] (visual set for
    positions < n_visual, text set after)."""
    return Dims(batch, n_q_heads, n_kv_heads, d_head, rank, max_seq, max_seqlen,
                DTYPE_CODE[io_dtype] if isinstance(io_dtype, str) else io_dtype,
                DTYPE_CODE[latent_dtype] if isinstance(latent_dtype, str) else latent_dtype,
                num_splits, ALGO_CODE[algo] if isinstance(algo, str) else algo, n_visual)


def plan(dims: Dims) -> dict:
    info = PlanInfo()
    rc = lib().lrkv_plan(ctypes.byref(dims), ctypes.byref(info))
    if rc:
        raise LrkvError("lrkv_plan", rc)
    return {"algo": {ALGO_SIMT: "simt", ALGO_TCGEN05: "tcgen05"}[info.algo],
            "num_splits": info.num_splits, "chunk": info.chunk, "grid": info.grid,
            "smem_bytes": info.smem_bytes, "full_chunk": info.full_chunk,
            "device_chunk": bool(info.device_chunk)}


def workspace_bytes(dims: Dims) -> int:
    n = lib().lrkv_workspace_bytes(ctypes.byref(dims))
    if n == 0:
        raise LrkvError("lrkv_workspace_bytes", -1)
    return n


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t: Optional[torch.Tensor], name: str, dtypes=None, numel=None, device=True):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if device and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtypes is not None and t.dtype not in dtypes:
        raise TypeError(f"{name} has dtype {t.dtype}, expected one of {dtypes}")
    if numel is not None and t.numel() != numel:
        raise ValueError(f"{name} has {t.numel()} elements, expected {numel}")
    return t.data_ptr()


def new_workspace(dims: Dims, device="cuda") -> torch.Tensor:
    """A zero-filled workspace of the size lrkv_workspace_bytes asks for."""
    return torch.zeros(workspace_bytes(dims), dtype=torch.uint8, device=device)


def _shapes(d: Dims):
    io = _TORCH_OF[d.io_dtype]
    return {
        "q": (d.batch * d.n_q_heads * d.d_head, (io,)),
        "Z": (d.batch * d.n_kv_heads * d.max_seq * d.rank, _LATENT_TORCH_OK[d.latent_dtype]),
        "S": (d.batch * d.n_kv_heads * d.max_seq, (torch.float32,)),
        "B": ((2 if d.n_visual > 0 else 1) * d.n_kv_heads * d.rank * d.d_head, (io,)),
        "znew": (d.batch * d.n_kv_heads * d.rank, (io,)),
        "seq": (d.batch, (torch.int32,)),
        "lse": (d.batch * d.n_q_heads, (torch.float32,)),
    }


def decode_attn(dims: Dims, q, ZK, ZV, ZK_scale, ZV_scale, BK, BV, seqlens, out,
                workspace, lse_out=None, stream=None) -> None:
    """lrkv_decode_attn: split-KV decode attention over the low-rank cache."""
    sh = _shapes(dims)
    args = [
        _ptr(q, "q", *sh["q"][::-1]), _ptr(ZK, "ZK", *sh["Z"][::-1]), _ptr(ZV, "ZV", *sh["Z"][::-1]),
        _ptr(ZK_scale, "ZK_scale", *sh["S"][::-1]), _ptr(ZV_scale, "ZV_scale", *sh["S"][::-1]),
        _ptr(BK, "BK", *sh["B"][::-1]), _ptr(BV, "BV", *sh["B"][::-1]),
        _ptr(seqlens, "seqlens", *sh["seq"][::-1]), _ptr(out, "out", *sh["q"][::-1]),
        _ptr(lse_out, "lse_out", *sh["lse"][::-1]), _ptr(workspace, "workspace")]
    rc = lib().lrkv_decode_attn(ctypes.byref(dims), *args, workspace.numel(), _stream(stream))
    if rc:
        raise LrkvError("lrkv_decode_attn", rc)


def decode_attn_shared(dims: Dims, q, ZK, ZV, ZK_scale, ZV_scale, DK, DV, seqlens, out,
                       workspace, lse_out=None, stream=None) -> None:
    """lrkv_decode_attn_shared: decode attention over a cross-head shared latent.
    ZK/ZV [B][max_seq][rank], scales [B][max_seq], DK/DV [rank][n_kv_heads * d_head]."""
    sh = _shapes(dims)
    io = sh["q"][1]
    nz = dims.batch * dims.max_seq * dims.rank
    nd = dims.rank * dims.n_kv_heads * dims.d_head
    ns = dims.batch * dims.max_seq
    args = [
        _ptr(q, "q", *sh["q"][::-1]), _ptr(ZK, "ZK", sh["Z"][1], nz), _ptr(ZV, "ZV", sh["Z"][1], nz),
        _ptr(ZK_scale, "ZK_scale", (torch.float32,), ns), _ptr(ZV_scale, "ZV_scale", (torch.float32,), ns),
        _ptr(DK, "DK", io, nd), _ptr(DV, "DV", io, nd),
        _ptr(seqlens, "seqlens", *sh["seq"][::-1]), _ptr(out, "out", *sh["q"][::-1]),
        _ptr(lse_out, "lse_out", *sh["lse"][::-1]), _ptr(workspace, "workspace")]
    rc = lib().lrkv_decode_attn_shared(ctypes.byref(dims), *args, workspace.numel(), _stream(stream))
    if rc:
        raise LrkvError("lrkv_decode_attn_shared", rc)


def decode_attn_adaptive(dims: Dims, q, ZK, ZV, ZK_scale, ZV_scale, BK, BV, seqlens,
                         importance, tau, r_low, beta, scores, out, lse_out, workspace,
                         stream=None) -> None:
    """lrkv_decode_attn_adaptive: decode attention with tokens below the importance
    threshold rebuilt at rank r_low, then importance <- beta * importance + (1 - beta) *
    attention mass. importance [B][Hkv][max_seq] and scores [B][Hq][max_seq] fp32."""
    sh = _shapes(dims)
    n_imp = dims.batch * dims.n_kv_heads * dims.max_seq
    n_sc = dims.batch * dims.n_q_heads * dims.max_seq
    args = [
        _ptr(q, "q", *sh["q"][::-1]), _ptr(ZK, "ZK", *sh["Z"][::-1]), _ptr(ZV, "ZV", *sh["Z"][::-1]),
        _ptr(ZK_scale, "ZK_scale", *sh["S"][::-1]), _ptr(ZV_scale, "ZV_scale", *sh["S"][::-1]),
        _ptr(BK, "BK", *sh["B"][::-1]), _ptr(BV, "BV", *sh["B"][::-1]),
        _ptr(seqlens, "seqlens", *sh["seq"][::-1]),
        _ptr(importance, "importance", (torch.float32,), n_imp)]
    rc = lib().lrkv_decode_attn_adaptive(
        ctypes.byref(dims), *args, float(tau), int(r_low), float(beta),
        _ptr(scores, "scores", (torch.float32,), n_sc), _ptr(out, "out", *sh["q"][::-1]),
        _ptr(lse_out, "lse_out", *sh["lse"][::-1]), _ptr(workspace, "workspace"),
        workspace.numel(), _stream(stream))
    if rc:
        raise LrkvError("lrkv_decode_attn_adaptive", rc)


def decode_attn_timed(dims: Dims, q, ZK, ZV, ZK_scale, ZV_scale, BK, BV, seqlens, out,
                      workspace, ev_begin, ev_end, lse_out=None, stream=None) -> None:
    """lrkv_decode_attn_timed: as decode_attn, recording two torch.cuda.Event (or raw
    cudaEvent_t handles) around the split kernel."""
    sh = _shapes(dims)
    args = [
        _ptr(q, "q", *sh["q"][::-1]), _ptr(ZK, "ZK", *sh["Z"][::-1]), _ptr(ZV, "ZV", *sh["Z"][::-1]),
        _ptr(ZK_scale, "ZK_scale", *sh["S"][::-1]), _ptr(ZV_scale, "ZV_scale", *sh["S"][::-1]),
        _ptr(BK, "BK", *sh["B"][::-1]), _ptr(BV, "BV", *sh["B"][::-1]),
        _ptr(seqlens, "seqlens", *sh["seq"][::-1]), _ptr(out, "out", *sh["q"][::-1]),
        _ptr(lse_out, "lse_out", *sh["lse"][::-1]), _ptr(workspace, "workspace")]
    evs = [getattr(e, "cuda_event", e) for e in (ev_begin, ev_end)]
    rc = lib().lrkv_decode_attn_timed(ctypes.byref(dims), *args, workspace.numel(),
                                      _stream(stream), *evs)
    if rc:
        raise LrkvError("lrkv_decode_attn_timed", rc)


NOALLOC_MAX_WORKSPACE_BYTES = 16 << 20


def decode_attn_noalloc(dims: Dims, q, ZK, ZV, ZK_scale, ZV_scale, BK, BV, seqlens, out,
                        lse_out=None, status_out=None, stream=None) -> None:
    """lrkv_decode_attn_noalloc: decode attention with the library's fixed scratch area
    (no workspace argument; for callers that cannot allocate device memory). Calls
    share one scratch area per device: do not let them overlap on the GPU."""
    sh = _shapes(dims)
    args = [
        _ptr(q, "q", *sh["q"][::-1]), _ptr(ZK, "ZK", *sh["Z"][::-1]), _ptr(ZV, "ZV", *sh["Z"][::-1]),
        _ptr(ZK_scale, "ZK_scale", *sh["S"][::-1]), _ptr(ZV_scale, "ZV_scale", *sh["S"][::-1]),
        _ptr(BK, "BK", *sh["B"][::-1]), _ptr(BV, "BV", *sh["B"][::-1]),
        _ptr(seqlens, "seqlens", *sh["seq"][::-1]), _ptr(out, "out", *sh["q"][::-1]),
        _ptr(lse_out, "lse_out", *sh["lse"][::-1]),
        _ptr(status_out, "status_out", (torch.int32,), 1)]
    rc = lib().lrkv_decode_attn_noalloc(ctypes.byref(dims), *args, _stream(stream))
    if rc:
        raise LrkvError("lrkv_decode_attn_noalloc", rc)


def debug_stall_next_launch(on: bool = True) -> None:
    """Test hook: the next tensor-core split launch withholds the first tile of work
    unit 0 so the waits on it run out (LRKV_STATUS_TIMEOUT); see
    lrkv_debug_stall_next_launch."""
    lib().lrkv_debug_stall_next_launch(1 if on else 0)


class PreparedStep:
    """One decode step (append, then attend) with every pointer checked once.

    Calling it issues lrkv_append and lrkv_decode_attn_timed on ``stream`` with the
    stored pointers: no per-call tensor inspection, so the host cost per step is two
    ctypes calls. The tensors must stay alive and in place.
    """

    def __init__(self, dims: Dims, q, ZK, ZV, ZK_scale, ZV_scale, BK, BV, seqlens, out,
                 workspace, zk_new, zv_new):
        sh = _shapes(dims)
        self.dims = dims
        self._keep = (q, ZK, ZV, ZK_scale, ZV_scale, BK, BV, seqlens, out, workspace, zk_new,
                      zv_new)
        self.attn_args = [
            _ptr(q, "q", *sh["q"][::-1]), _ptr(ZK, "ZK", *sh["Z"][::-1]),
            _ptr(ZV, "ZV", *sh["Z"][::-1]), _ptr(ZK_scale, "ZK_scale", *sh["S"][::-1]),
            _ptr(ZV_scale, "ZV_scale", *sh["S"][::-1]), _ptr(BK, "BK", *sh["B"][::-1]),
            _ptr(BV, "BV", *sh["B"][::-1]), _ptr(seqlens, "seqlens", *sh["seq"][::-1]),
            _ptr(out, "out", *sh["q"][::-1]), None, _ptr(workspace, "workspace")]
        self.append_args = [
            _ptr(zk_new, "zk_new", *sh["znew"][::-1]), _ptr(zv_new, "zv_new", *sh["znew"][::-1]),
            self.attn_args[1], self.attn_args[2], self.attn_args[3], self.attn_args[4],
            self.attn_args[7], self.attn_args[10]]
        self.ws_bytes = workspace.numel()

    def __call__(self, stream, ev_begin=None, ev_end=None):
        L = lib()
        rc = L.lrkv_append(ctypes.byref(self.dims), *self.append_args, self.ws_bytes, stream)
        if rc:
            raise LrkvError("lrkv_append", rc)
        rc = L.lrkv_decode_attn_timed(ctypes.byref(self.dims), *self.attn_args, self.ws_bytes,
                                      stream, ev_begin, ev_end)
        if rc:
            raise LrkvError("lrkv_decode_attn_timed", rc)


def append(dims: Dims, zk_new, zv_new, ZK, ZV, ZK_scale, ZV_scale, seqlens, workspace,
           stream=None) -> None:
    """lrkv_append: write one latent row per (b, KV head) at seqlens[b], then +1."""
    sh = _shapes(dims)
    args = [_ptr(zk_new, "zk_new", *sh["znew"][::-1]), _ptr(zv_new, "zv_new", *sh["znew"][::-1]),
            _ptr(ZK, "ZK", *sh["Z"][::-1]), _ptr(ZV, "ZV", *sh["Z"][::-1]),
            _ptr(ZK_scale, "ZK_scale", *sh["S"][::-1]), _ptr(ZV_scale, "ZV_scale", *sh["S"][::-1]),
            _ptr(seqlens, "seqlens", *sh["seq"][::-1]), _ptr(workspace, "workspace")]
    rc = lib().lrkv_append(ctypes.byref(dims), *args, workspace.numel(), _stream(stream))
    if rc:
        raise LrkvError("lrkv_append", rc)


def project_append(dims: Dims, x, AK, AV, ZK, ZV, ZK_scale, ZV_scale, seqlens, workspace,
                   stream=None) -> None:
    """lrkv_project_append: z = x A_g for every (b, KV head), written at seqlens[b] as
    lrkv_append writes a row, then seqlens[b] += 1. x [B][d_model], A [Hkv][d_model][r]."""
    sh = _shapes(dims)
    io = sh["q"][1]
    d_model = x.numel() // dims.batch if x is not None else 0
    args = [_ptr(x, "x", io, dims.batch * d_model),
            _ptr(AK, "AK", io, dims.n_kv_heads * d_model * dims.rank),
            _ptr(AV, "AV", io, dims.n_kv_heads * d_model * dims.rank),
            _ptr(ZK, "ZK", *sh["Z"][::-1]), _ptr(ZV, "ZV", *sh["Z"][::-1]),
            _ptr(ZK_scale, "ZK_scale", *sh["S"][::-1]), _ptr(ZV_scale, "ZV_scale", *sh["S"][::-1]),
            _ptr(seqlens, "seqlens", *sh["seq"][::-1]), _ptr(workspace, "workspace")]
    rc = lib().lrkv_project_append(ctypes.byref(dims), d_model, *args, workspace.numel(),
                                   _stream(stream))
    if rc:
        raise LrkvError("lrkv_project_append", rc)


def decode_step_host(dims: Dims, q_host, zk_new_host, zv_new_host, out_host, q_dev, zk_new_dev,
                     zv_new_dev, out_dev, ZK, ZV, ZK_scale, ZV_scale, BK, BV, seqlens,
                     workspace, stream=None) -> None:
    """lrkv_decode_step_host: H2D copies, append, attend, D2H copy, on one stream."""
    sh = _shapes(dims)
    host = [_ptr(q_host, "q_host", sh["q"][1], sh["q"][0], device=False),
            _ptr(zk_new_host, "zk_new_host", sh["znew"][1], sh["znew"][0], device=False),
            _ptr(zv_new_host, "zv_new_host", sh["znew"][1], sh["znew"][0], device=False),
            _ptr(out_host, "out_host", sh["q"][1], sh["q"][0], device=False)]
    dev = [_ptr(q_dev, "q_dev", *sh["q"][::-1]), _ptr(zk_new_dev, "zk_new_dev", *sh["znew"][::-1]),
           _ptr(zv_new_dev, "zv_new_dev", *sh["znew"][::-1]), _ptr(out_dev, "out_dev", *sh["q"][::-1]),
           _ptr(ZK, "ZK", *sh["Z"][::-1]), _ptr(ZV, "ZV", *sh["Z"][::-1]),
           _ptr(ZK_scale, "ZK_scale", *sh["S"][::-1]), _ptr(ZV_scale, "ZV_scale", *sh["S"][::-1]),
           _ptr(BK, "BK", *sh["B"][::-1]), _ptr(BV, "BV", *sh["B"][::-1]),
           _ptr(seqlens, "seqlens", *sh["seq"][::-1]), _ptr(workspace, "workspace")]
    rc = lib().lrkv_decode_step_host(ctypes.byref(dims), *host, *dev, workspace.numel(),
                                     _stream(stream))
    if rc:
        raise LrkvError("lrkv_decode_step_host", rc)


def read_status(workspace, stream=None) -> int:
    """lrkv_read_status: synchronise, return and clear the device status word."""
    v = ctypes.c_uint32(0)
    rc = lib().lrkv_read_status(_ptr(workspace, "workspace"), _stream(stream), ctypes.byref(v))
    if rc:
        raise LrkvError("lrkv_read_status", rc)
    return v.value


def workspace_init(workspace, stream=None) -> None:
    rc = lib().lrkv_workspace_init(_ptr(workspace, "workspace"), workspace.numel(), _stream(stream))
    if rc:
        raise LrkvError("lrkv_workspace_init", rc)
