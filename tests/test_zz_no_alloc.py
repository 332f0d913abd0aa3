"""The allocation-free entry point, lrkv_decode_attn_noalloc, for callers that cannot
allocate device memory themselves (a host program without a device memory manager,
or a runtime whose memory budget forbids allocations while it serves). It must give
the same results as lrkv_decode_attn, which uses a caller-provided workspace, on two
calls in a row (the second reuses the scratch left by the first). Collected last so
that a run stopping at the first failure has already run every other test; it also
passes on its own in a fresh process."""
import numpy as np
import pytest
import torch

from rank_kv_cache_head_b200 import lrkv
from rank_kv_cache_head_b200.workloads import WORKLOADS, make_inputs

from helpers import TOL_LOWP_MAXABS, TOL_LOWP_RELL2, dims_for, to_device

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["vlm7b-bf16", "quant-i8"])
def test_noalloc_matches_workspace_entry_point_twice(name):
    wl = WORKLOADS[name].scaled(batch=3, seq_len=1500, seed=77)
    inputs = make_inputs(wl, capacity=1536)
    dims = dims_for(wl, inputs)
    assert lrkv.workspace_bytes(dims) <= lrkv.NOALLOC_MAX_WORKSPACE_BYTES
    dev = to_device(inputs)
    ref = torch.empty_like(dev["q"])
    ref_lse = torch.empty(wl.batch, wl.n_q_heads, device="cuda")
    ws = lrkv.new_workspace(dims)
    lrkv.decode_attn(dims, dev["q"], dev["ZK"], dev["ZV"], dev["ZK_scale"], dev["ZV_scale"],
                     dev["BK"], dev["BV"], dev["seqlens"], ref, ws, lse_out=ref_lse)
    assert lrkv.read_status(ws) == 0
    r = ref.double().cpu().numpy()
    for call in range(2):
        out = torch.full_like(dev["q"], float("nan"))
        lse = torch.full((wl.batch, wl.n_q_heads), float("nan"), device="cuda")
        status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
        lrkv.decode_attn_noalloc(dims, dev["q"], dev["ZK"], dev["ZV"], dev["ZK_scale"],
                                 dev["ZV_scale"], dev["BK"], dev["BV"], dev["seqlens"], out,
                                 lse_out=lse, status_out=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0, f"call {call}: device status {int(status.item())}"
        o = out.double().cpu().numpy()
        assert np.all(np.isfinite(o)), f"call {call}: non-finite output"
        err = np.abs(o - r)
        assert err.max() <= TOL_LOWP_MAXABS, f"call {call}: max-abs {err.max():.3e}"
        rel = np.linalg.norm(o - r) / np.linalg.norm(r)
        assert rel <= TOL_LOWP_RELL2, f"call {call}: rel-L2 {rel:.3e}"
        assert np.allclose(lse.cpu().numpy(), ref_lse.cpu().numpy(), atol=1e-3, rtol=0)


def test_noalloc_rejects_sizes_above_its_maximum():
    """A problem whose workspace exceeds the fixed scratch area is refused with
    LRKV_ERR_WORKSPACE before anything is launched (the pointers are never read)."""
    dims = lrkv.make_dims(512, 32, 8, 128, 48, 4096, 4096, "bf16", "bf16", 64)
    assert lrkv.workspace_bytes(dims) > lrkv.NOALLOC_MAX_WORKSPACE_BYTES
    fake = [0x10000 + 256 * i for i in range(9)]
    rc = lrkv.lib().lrkv_decode_attn_noalloc(lrkv.ctypes.byref(dims), *fake, None, None, None)
    assert rc == -4 and lrkv.strerror(rc) == "workspace missing or too small"
