"""The N > 1 path on CPU: two gloo ranks.

Decode attention shards by (batch row, KV head) with no exchange step, so a multi-GPU
run is independent ranks plus the bench's timing reductions (the max of the ranks'
times, the sum of their bytes). These tests run two processes over gloo: the bench's
rank set-up and reductions, and a batch split across ranks whose per-rank results,
put side by side, equal the unsplit result (computed with the oracle, on CPU)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      LOCAL_RANK=str(rank), WORLD_SIZE=str(world))
    import torch.distributed as dist

    import bench
    from oracle import lrkv_oracle as orc
    from rank_kv_cache_head_b200.metrics import max_over_ranks, sum_over_ranks
    from rank_kv_cache_head_b200.workloads import WORKLOADS, make_inputs
    try:
        r, w, local = bench.dist_init()
        assert (r, w, local) == (rank, world, rank) and dist.get_backend() == "gloo"
        mx = max_over_ranks(float(rank + 1))
        sm = sum_over_ranks(float(10 * (rank + 1)))
        # this rank's shard of the batch: rows rank, rank + world, ...
        wl = WORKLOADS["tiny-fp32"].scaled(batch=4, seq_len=40, seed=5)
        x = make_inputs(wl, capacity=40)
        rows = list(range(rank, wl.batch, world))
        f = lambda t: t.numpy().astype(np.float64)
        out, lse = orc.decode_attention(f(x["q"])[rows], f(x["ZK"])[rows], f(x["ZV"])[rows],
                                        f(x["BK"]), f(x["BV"]), x["seqlens"].numpy()[rows])
        bench.barrier()
        q.put((rank, mx, sm, rows, out, lse))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


@pytest.mark.timeout(300)
def test_two_gloo_ranks_reduce_and_shard():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=240) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort(key=lambda t: t[0])
    assert all(t[1] == 2.0 for t in res)           # max over ranks
    assert all(t[2] == 30.0 for t in res)          # sum over ranks
    from oracle import lrkv_oracle as orc
    from rank_kv_cache_head_b200.workloads import WORKLOADS, make_inputs
    wl = WORKLOADS["tiny-fp32"].scaled(batch=4, seq_len=40, seed=5)
    x = make_inputs(wl, capacity=40)
    f = lambda t: t.numpy().astype(np.float64)
    ref_out, ref_lse = orc.decode_attention(f(x["q"]), f(x["ZK"]), f(x["ZV"]), f(x["BK"]),
                                            f(x["BV"]), x["seqlens"].numpy())
    for _, _, _, rows, out, lse in res:
        np.testing.assert_array_equal(out, ref_out[rows])
        np.testing.assert_array_equal(lse, ref_lse[rows])
