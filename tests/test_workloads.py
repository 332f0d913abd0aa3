"""CPU checks of the seeded input generator (shapes, dtypes, layout, recipe)."""
import numpy as np
import pytest
import torch

from rank_kv_cache_head_b200.workloads import WORKLOADS, make_append_rows, make_inputs, sigmas


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_small_versions_are_contiguous_and_typed(name):
    wl = WORKLOADS[name].scaled(batch=2, seq_len=300, ragged_min=None if
                                WORKLOADS[name].ragged_min is None else 100)
    x = make_inputs(wl, capacity=320)
    for k, v in x.items():
        if v is not None:
            assert v.is_contiguous(), k
    assert x["q"].shape == (2, wl.n_q_heads, wl.d_head)
    assert x["ZK"].shape == (2, wl.n_kv_heads, 320, wl.rank)
    assert x["BK"].shape == (wl.n_kv_heads, wl.rank, wl.d_head)
    assert (x["ZK_scale"] is not None) == (wl.latent_dtype in ("i8", "e4m3"))
    rows = make_append_rows(wl)
    assert rows["zk_new"].shape == (2, wl.n_kv_heads, wl.rank) and rows["zk_new"].is_contiguous()


def test_factor_rows_are_orthonormal_times_sigma():
    wl = WORKLOADS["longvideo-bf16"].scaled(batch=1, seq_len=64, io_dtype="f32", latent_dtype="f32")
    x = make_inputs(wl)
    sig = sigmas(wl)
    B = x["BK"][0].double().numpy()
    gram = B @ B.T
    assert np.allclose(gram, np.diag(sig ** 2), atol=1e-6)


def test_text_factor_set_is_a_second_draw_of_the_same_recipe():
    from rank_kv_cache_head_b200.workloads import with_text_factors
    wl = WORKLOADS["vlm7b-bf16"].scaled(batch=1, seq_len=64, n_q_heads=2, n_kv_heads=2,
                                        io_dtype="f32", latent_dtype="f32")
    x = make_inputs(wl)
    m = with_text_factors(wl, x)
    assert m["BK"].shape == (2, 2, wl.rank, wl.d_head) and m["BK"].is_contiguous()
    assert torch.equal(m["BK"][0], x["BK"]) and torch.equal(m["BV"][0], x["BV"])
    assert not torch.equal(m["BK"][1], x["BK"]) and not torch.equal(m["BK"][1], m["BV"][1])
    sig = sigmas(wl)
    for k in ("BK", "BV"):
        T = m[k][1][1].double().numpy()
        assert np.allclose(T @ T.T, np.diag(sig ** 2), atol=1e-6)
    assert m["ZK"] is x["ZK"]


def test_outlier_positions_scaled():
    wl = WORKLOADS["longvideo-bf16"].scaled(batch=1, seq_len=1000, io_dtype="f32",
                                            latent_dtype="f32")
    x = make_inputs(wl)
    norms = x["ZK"][0].double().norm(dim=-1).mean(dim=0).numpy()  # per position
    big = norms > 4 * np.median(norms)
    assert big.sum() == 10   # floor(1% of 1000), shared by all heads


def test_ragged_lengths_in_range_and_seeded():
    wl = WORKLOADS["gqa-ragged-bf16"]
    from rank_kv_cache_head_b200.workloads import seqlens_for
    a, b = seqlens_for(wl), seqlens_for(wl)
    assert np.array_equal(a, b) and a.min() >= 128 and a.max() <= 4096 and len(a) == 64
