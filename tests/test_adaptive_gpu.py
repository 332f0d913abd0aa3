"""GPU parity of the attention-aware partial decompression (lrkv_decode_attn_adaptive)
against the oracle: outputs and LSE within the decode tolerances, the updated
importance within fp32 rounding of the oracle's moving average on every attended
position and bit-identical elsewhere; with every token important the output is
bit-identical to the plain CUDA-core decode."""
import numpy as np
import pytest
import torch

from oracle import lrkv_oracle as orc
from rank_kv_cache_head_b200 import lrkv
from rank_kv_cache_head_b200.workloads import WORKLOADS, make_inputs, with_text_factors

from helpers import compare, oracle_inputs, to_device

pytestmark = pytest.mark.gpu

CASES = {
    "vlm-small": (WORKLOADS["vlm7b-bf16"].scaled(batch=2, n_q_heads=4, n_kv_heads=4, seq_len=700,
                                                 seed=51), 0),
    "gqa-ragged-small": (WORKLOADS["gqa-ragged-bf16"].scaled(batch=5, n_q_heads=8, n_kv_heads=2,
                                                             seq_len=900, ragged_min=1, seed=52), 0),
    "quant-i8-small": (WORKLOADS["quant-i8"].scaled(batch=3, n_q_heads=8, n_kv_heads=2,
                                                    seq_len=600, seed=53), 0),
    "tiny-fp32": (WORKLOADS["tiny-fp32"].scaled(batch=2, ragged_min=20, seed=54), 0),
    "vlm-modal": (WORKLOADS["vlm7b-bf16"].scaled(batch=2, n_q_heads=4, n_kv_heads=2, seq_len=700,
                                                 seed=55), 576),
}


def _setup(wl, P, seed=0):
    x = make_inputs(wl)
    if P:
        x = with_text_factors(wl, x)
    rng = np.random.default_rng(seed)
    imp = rng.uniform(0.0, 1.0, (wl.batch, wl.n_kv_heads, x["ZK"].shape[2])).astype(np.float32)
    dims = lrkv.make_dims(wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.d_head, wl.rank,
                          x["ZK"].shape[2], int(x["seqlens"].max()), wl.io_dtype, wl.latent_dtype,
                          0, "simt", n_visual=P)
    return x, imp, dims


def _run(wl, x, imp, dims, tau, r_low, beta):
    dev = to_device(x)
    io_t = torch.float32 if wl.io_dtype == "f32" else torch.bfloat16
    out = torch.empty((wl.batch, wl.n_q_heads, wl.d_head), dtype=io_t, device="cuda")
    lse = torch.empty((wl.batch, wl.n_q_heads), dtype=torch.float32, device="cuda")
    imp_d = torch.from_numpy(imp.copy()).cuda()
    scores = torch.empty((wl.batch, wl.n_q_heads, x["ZK"].shape[2]), dtype=torch.float32,
                         device="cuda")
    ws = lrkv.new_workspace(dims)
    lrkv.decode_attn_adaptive(dims, dev["q"], dev["ZK"], dev["ZV"], dev["ZK_scale"], dev["ZV_scale"],
                              dev["BK"], dev["BV"], dev["seqlens"], imp_d, tau, r_low, beta, scores,
                              out, lse, ws)
    return (out.double().cpu().numpy(), lse.cpu().numpy().astype(np.float64),
            imp_d.cpu().numpy(), lrkv.read_status(ws))


@pytest.mark.parametrize("name", list(CASES))
def test_adaptive_parity(name):
    wl, P = CASES[name]
    x, imp, dims = _setup(wl, P, seed=1)
    tau, r_low, beta = 0.5, max(1, wl.rank // 4), 0.8
    out, lse, new_imp, status = _run(wl, x, imp, dims, tau, r_low, beta)
    assert status == 0
    o = oracle_inputs(wl, x)
    ref, ref_lse, _, ref_imp = orc.decode_attention_adaptive(
        o["q"], o["ZK"], o["ZV"], o["BK"], o["BV"], o["seqlens"], imp, tau, r_low, beta,
        o["ZK_scale"], o["ZV_scale"], n_visual=P)
    compare(wl, out, ref, lse, ref_lse)
    G = wl.n_q_heads // wl.n_kv_heads
    for b, L in enumerate(x["seqlens"].numpy()):
        np.testing.assert_allclose(new_imp[b, :, :L], ref_imp[b, :, :L], rtol=2e-4, atol=2e-5 * G)
        np.testing.assert_array_equal(new_imp[b, :, L:], imp[b, :, L:])
    # the reduced rank really changes the result on this input
    full, _ = orc.decode_attention(o["q"], o["ZK"], o["ZV"], o["BK"], o["BV"], o["seqlens"],
                                   o["ZK_scale"], o["ZV_scale"], n_visual=P)
    assert np.linalg.norm(full - ref) > 10 * 5e-3 * np.linalg.norm(ref)


def test_all_important_is_the_plain_kernel_bit_for_bit():
    wl, P = CASES["gqa-ragged-small"]
    x, imp, dims = _setup(wl, P, seed=2)
    out, lse, _, status = _run(wl, x, imp, dims, -np.inf, 1, 0.5)
    assert status == 0
    dev = to_device(x)
    plain = torch.empty((wl.batch, wl.n_q_heads, wl.d_head), dtype=torch.bfloat16, device="cuda")
    plain_lse = torch.empty((wl.batch, wl.n_q_heads), dtype=torch.float32, device="cuda")
    ws = lrkv.new_workspace(dims)
    lrkv.decode_attn(dims, dev["q"], dev["ZK"], dev["ZV"], None, None, dev["BK"], dev["BV"],
                     dev["seqlens"], plain, ws, lse_out=plain_lse)
    assert np.array_equal(out, plain.double().cpu().numpy())
    assert np.array_equal(lse, plain_lse.cpu().numpy().astype(np.float64))


def test_tensor_core_request_is_refused():
    wl, P = CASES["vlm-small"]
    x, imp, _ = _setup(wl, P)
    dims = lrkv.make_dims(wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.d_head, wl.rank,
                          x["ZK"].shape[2], int(x["seqlens"].max()), wl.io_dtype, wl.latent_dtype,
                          0, "tcgen05")
    with pytest.raises(lrkv.LrkvError) as e:
        _run(wl, x, imp, dims, 0.5, 4, 0.5)
    assert e.value.code == -6   # LRKV_ERR_UNSUPPORTED
