"""The bounded-wait error path of the tensor-core split kernel, forced on purpose.

With lrkv_debug_stall_next_launch, the producer that takes work unit 0 withholds that
unit's first latent tile (no copy, no arrival): the waits on that tile run out after
their one-second bound, the CTA unwinds (drains its copies, waits for its MMAs, frees
tensor memory) and the launch reports LRKV_STATUS_TIMEOUT through the workspace status
word. The next launch on the same context must then be correct: nothing faulted or
hung."""
import pytest

from rank_kv_cache_head_b200 import lrkv
from rank_kv_cache_head_b200.workloads import WORKLOADS, make_inputs

from helpers import compare, dims_for, run_gpu, run_oracle, to_device

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["vlm7b-bf16", "quant-i8"])
def test_withheld_tile_times_out_and_context_survives(name):
    wl = WORKLOADS[name].scaled(batch=2, seq_len=1000, seed=41)
    inputs = make_inputs(wl, capacity=1024)
    assert lrkv.plan(dims_for(wl, inputs, algo="tcgen05"))["algo"] == "tcgen05"
    dev = to_device(inputs)
    lrkv.debug_stall_next_launch(True)
    _, _, status, _ = run_gpu(wl, inputs, algo="tcgen05", dev=dev)
    assert status & lrkv.STATUS_TIMEOUT, f"status {status}"
    out, lse, status, _ = run_gpu(wl, inputs, algo="tcgen05", dev=dev)
    assert status == 0
    ref, ref_lse = run_oracle(wl, inputs)
    compare(wl, out, ref, lse, ref_lse)
