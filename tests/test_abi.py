"""CPU checks of the C ABI: the library loads, exports every function the headers in
include/ declare, and validates arguments (no compute call is made without a GPU)."""
import ctypes
import os
import re

import pytest

from rank_kv_cache_head_b200 import lrkv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = sorted(os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include"))
                 if f.endswith(".h"))


def declared_functions():
    src = "".join(open(h).read() for h in HEADERS)
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(lrkv_[a-z_0-9]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("lrkv_decode_attn", "lrkv_append", "lrkv_workspace_bytes",
                     "lrkv_read_status", "lrkv_strerror", "lrkv_project_append",
                     "lrkv_decode_attn_adaptive", "lrkv_decode_attn_shared"):
        assert required in names


def test_library_exports_every_declared_function():
    L = lrkv.lib()
    missing = [n for n in declared_functions() if not hasattr(L, n)]
    assert not missing, missing
    assert lrkv.version() == 2


def test_strerror_codes():
    assert lrkv.strerror(0) == "success"
    for c in range(-1, -8, -1):
        assert lrkv.strerror(c) != "unknown error"


def _dims(**kw):
    base = dict(batch=2, n_q_heads=8, n_kv_heads=2, d_head=128, rank=32, max_seq=1024,
                max_seqlen=1000, io_dtype="bf16", latent_dtype="bf16")
    base.update(kw)
    return lrkv.make_dims(**base)


def _plan_rc(d):
    info = lrkv.PlanInfo()
    return lrkv.lib().lrkv_plan(ctypes.byref(d), ctypes.byref(info))


@pytest.mark.parametrize("kw,code", [
    (dict(n_q_heads=6, n_kv_heads=4), -1),
    (dict(d_head=96), -1),
    (dict(rank=12), -1),
    (dict(rank=264), -1),
    (dict(max_seqlen=2000), -1),
    (dict(max_seq=0, max_seqlen=0), -1),
    (dict(io_dtype="i8"), -2),
    (dict(io_dtype="bf16", latent_dtype="f32"), -2),
    (dict(latent_dtype="i8", rank=8), -3),
    (dict(num_splits=-1), -1),
    (dict(n_visual=8), -1),             # modality boundary not a multiple of 16
    (dict(n_visual=-16), -1),
    (dict(n_visual=4096), -1),          # past the capacity
])
def test_invalid_dims_rejected(kw, code):
    assert _plan_rc(_dims(**kw)) == code
    assert lrkv.lib().lrkv_workspace_bytes(ctypes.byref(_dims(**kw))) == 0


def test_plan_and_workspace_sizes():
    d = _dims()
    p = lrkv.plan(d)
    assert p["chunk"] % 128 == 0 and p["num_splits"] * p["chunk"] >= 1000
    ws = lrkv.workspace_bytes(d)
    parts = 2 * 8 * p["num_splits"]
    assert ws >= 256 + parts * 4 + parts * 128 * 4
    # explicit split counts are honoured (clamped to the tile count)
    for s in (1, 2, 3, 8, 100):
        p = lrkv.plan(_dims(num_splits=s))
        assert p["num_splits"] == min(s, 8) or p["num_splits"] * p["chunk"] >= 1000
        assert (p["num_splits"] - 1) * p["chunk"] < 1000


def test_null_and_alignment_errors_do_not_launch():
    d = _dims()
    L = lrkv.lib()
    # NULL required pointers -> LRKV_ERR_ARG before any CUDA call
    rc = L.lrkv_decode_attn(ctypes.byref(d), *([None] * 11), 0, None)
    assert rc == -7
    rc = L.lrkv_append(ctypes.byref(d), *([None] * 8), 0, None)
    assert rc == -7
    # misaligned (fake, never dereferenced) pointers -> LRKV_ERR_ALIGN
    fake = [0x1000 + 8 * (i == 0) for i in range(11)]
    fake[3] = fake[4] = None  # no scales for bf16 latents
    fake[9] = None
    rc = L.lrkv_decode_attn(ctypes.byref(d), *fake, 1 << 30, None)
    assert rc == -3
    # workspace too small -> LRKV_ERR_WORKSPACE
    fake[0] = 0x1000
    rc = L.lrkv_decode_attn(ctypes.byref(d), *fake, 16, None)
    assert rc == -4
    # scales required exactly for quantised latents
    dq = _dims(latent_dtype="i8")
    rc = L.lrkv_decode_attn(ctypes.byref(dq), *fake, 1 << 30, None)
    assert rc == -7


def test_binding_refuses_cpu_tensors():
    import torch
    d = _dims()
    t = torch.zeros(4)
    with pytest.raises((ValueError, TypeError)):
        lrkv.decode_attn(d, t, t, t, None, None, t, t, t, t, t)


def test_adaptive_arguments_checked_before_any_launch():
    """lrkv_decode_attn_adaptive refuses the tensor-core kernel, NULL state buffers and
    out-of-range rank or decay before touching the device."""
    L = lrkv.lib()
    d = _dims()
    fake = ctypes.c_void_p(16)

    def call(dims, imp=fake, scores=fake, lse=fake, r_low=8, beta=0.5):
        return L.lrkv_decode_attn_adaptive(ctypes.byref(dims), fake, fake, fake, None, None, fake,
                                           fake, fake, imp, 0.5, r_low, beta, scores, fake, lse,
                                           fake, 1 << 20, None)
    assert call(_dims(algo="tcgen05")) == -6
    assert call(d, imp=None) == -7
    assert call(d, scores=None) == -7
    assert call(d, lse=None) == -7
    assert call(d, r_low=0) == -7
    assert call(d, r_low=33) == -7
    assert call(d, beta=1.5) == -7
    assert call(d, beta=float("nan")) == -7
    assert call(_dims(rank=12)) == -1


def test_shared_latent_arguments_checked_before_any_launch():
    L = lrkv.lib()
    fake = ctypes.c_void_p(16)

    def call(dims):
        return L.lrkv_decode_attn_shared(ctypes.byref(dims), fake, fake, fake, None, None, fake,
                                         fake, fake, fake, None, fake, 1 << 20, None)
    assert call(_dims(algo="tcgen05")) == -6
    assert call(_dims(n_visual=16)) == -1
    assert call(_dims(rank=12)) == -1
