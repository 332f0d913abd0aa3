"""Split sizes chosen on the device (automatic splitting on the tensor-core path).

The host plans the split size for rows at full length (full_chunk) and sizes the
workspace for the finest split allowed (chunk); the kernel's producer scales
full_chunk by the share of 128-token tiles the rows actually hold, clamped to
[chunk, full_chunk], and records its choice in header word 4 for the merge. These
tests check the recorded choice against that rule evaluated here from the lengths,
and the result against the oracle, for ragged, short and full-length batches."""
import numpy as np
import pytest
import torch

from rank_kv_cache_head_b200 import lrkv
from rank_kv_cache_head_b200.workloads import WORKLOADS, make_inputs

from helpers import compare, dims_for, run_gpu, run_oracle, to_device

pytestmark = pytest.mark.gpu


def _expected_chunk(plan, seqlens, max_seqlen):
    tiles_max = max(1, -(-max_seqlen // 128))
    tiles = int(sum(-(-int(L) // 128) for L in seqlens))
    full = len(seqlens) * tiles_max
    hint = plan["full_chunk"] // 128
    ct = -(-hint * tiles // full)
    ct = max(plan["chunk"] // 128, min(ct, hint))
    return ct * 128


@pytest.mark.parametrize("name,lengths", [
    ("gqa-ragged-bf16", "half-short"),   # half the rows at 128 tokens
    ("gqa-ragged-bf16", "ragged"),       # the workload's own U[128, L] draw
    ("vlm7b-bf16", "full"),              # every row at max_seqlen: the host's choice
    ("quant-i8", "one-long"),            # one long row, the rest short
])
def test_device_chunk_matches_rule_and_oracle(name, lengths):
    L = 2048
    base = WORKLOADS[name].scaled(batch=12, seq_len=L, seed=88)
    rng = np.random.default_rng(5)
    if lengths == "half-short":
        seq = np.where(np.arange(base.batch) % 2 == 0, L, 128)
    elif lengths == "ragged":
        seq = rng.integers(128, L + 1, size=base.batch)
    elif lengths == "full":
        seq = np.full(base.batch, L)
    else:
        seq = np.full(base.batch, 130)
        seq[3] = L
    inputs = make_inputs(base, capacity=L, seqlens=seq.astype(np.int32))
    dims = dims_for(base, inputs, max_seqlen=L)
    plan = lrkv.plan(dims)
    assert plan["algo"] == "tcgen05"
    if not plan["device_chunk"]:
        # nothing to scale: the host's full-length split is already the finest
        assert plan["full_chunk"] == plan["chunk"] == 128
        pytest.skip("single-tile split planned for full-length rows")
    assert plan["chunk"] <= plan["full_chunk"] and plan["chunk"] % 128 == 0
    ws = lrkv.new_workspace(dims)
    out, lse, status, _ = run_gpu(base, inputs, max_seqlen=L, dev=to_device(inputs), ws=ws)
    assert status == 0
    chosen = int(ws[16:20].view(torch.int32).item())
    assert chosen == _expected_chunk(plan, seq, L)
    if lengths == "full":
        assert chosen == plan["full_chunk"]
    ref, ref_lse = run_oracle(base, inputs)
    compare(base, out, ref, lse, ref_lse)


def test_explicit_splits_are_not_rescaled():
    wl = WORKLOADS["gqa-ragged-bf16"].scaled(batch=4, seq_len=1024, seed=3)
    inputs = make_inputs(wl, capacity=1024)
    plan = lrkv.plan(dims_for(wl, inputs, num_splits=3, max_seqlen=1024))
    assert not plan["device_chunk"] and plan["num_splits"] == 3
    out, lse, status, _ = run_gpu(wl, inputs, num_splits=3, max_seqlen=1024)
    assert status == 0
    ref, ref_lse = run_oracle(wl, inputs)
    compare(wl, out, ref, lse, ref_lse)
