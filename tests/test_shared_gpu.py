"""GPU parity of decode attention over a cross-head shared latent
(lrkv_decode_attn_shared: one latent row per token for every KV head, one
decompression matrix [R][H_kv d]) against the oracle, on bf16, int8 and fp32 caches
with ragged lengths, and with automatic and explicit split counts."""
import numpy as np
import pytest
import torch

from oracle import lrkv_oracle as orc
from rank_kv_cache_head_b200 import lrkv
from rank_kv_cache_head_b200.workloads import WORKLOADS

from helpers import compare

pytestmark = pytest.mark.gpu


def _case(wl, R, seed):
    """Seeded shared-latent inputs in the workload's stored dtypes."""
    rng = np.random.default_rng(seed)
    B, Hq, Hkv, d, L = wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.d_head, wl.seq_len
    io_t = torch.float32 if wl.io_dtype == "f32" else torch.bfloat16
    q = torch.from_numpy(rng.standard_normal((B, Hq, d))).to(io_t)
    D = [torch.from_numpy(rng.standard_normal((R, Hkv * d)) / np.sqrt(R)).to(io_t) for _ in range(2)]
    seq = rng.integers(1, L + 1, size=B).astype(np.int32)
    seq[0] = L
    quant = wl.latent_dtype == "i8"
    if quant:
        Z = [torch.from_numpy(np.clip(np.rint(rng.standard_normal((B, L, R)) * 40), -127, 127)).to(torch.int8)
             for _ in range(2)]
        S = [torch.from_numpy(rng.uniform(0.01, 0.03, (B, L)).astype(np.float32)) for _ in range(2)]
    else:
        zt = torch.float32 if wl.latent_dtype == "f32" else torch.bfloat16
        Z = [torch.from_numpy(rng.standard_normal((B, L, R))).to(zt) for _ in range(2)]
        S = [None, None]
    return q, Z, S, D, torch.from_numpy(seq)


def _f64(t):
    return None if t is None else t.double().numpy()


@pytest.mark.parametrize("name,R", [("vlm7b-bf16", 64), ("quant-i8", 64), ("tiny-fp32", 32)])
@pytest.mark.parametrize("num_splits", [0, 3])
def test_shared_latent_parity(name, R, num_splits):
    wl = WORKLOADS[name].scaled(batch=3, n_q_heads=8, n_kv_heads=4, seq_len=520, seed=61)
    if name == "tiny-fp32":
        wl = wl.scaled(n_q_heads=4, n_kv_heads=2)
    q, Z, S, D, seq = _case(wl, R, 70 + R)
    dims = lrkv.make_dims(wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.d_head, R, wl.seq_len,
                          wl.seq_len, wl.io_dtype, wl.latent_dtype, num_splits, "simt")
    io_t = q.dtype
    out = torch.empty((wl.batch, wl.n_q_heads, wl.d_head), dtype=io_t, device="cuda")
    lse = torch.empty((wl.batch, wl.n_q_heads), dtype=torch.float32, device="cuda")
    ws = lrkv.new_workspace(dims)
    cu = lambda t: None if t is None else t.cuda()
    lrkv.decode_attn_shared(dims, q.cuda(), cu(Z[0]), cu(Z[1]), cu(S[0]), cu(S[1]), cu(D[0]),
                            cu(D[1]), seq.cuda(), out, ws, lse_out=lse)
    assert lrkv.read_status(ws) == 0
    ref, ref_lse = orc.decode_attention_shared(_f64(q), _f64(Z[0]), _f64(Z[1]), _f64(D[0]), _f64(D[1]),
                                               seq.numpy(), wl.n_kv_heads, _f64(S[0]), _f64(S[1]))
    compare(wl, out.double().cpu().numpy(), ref, lse.cpu().numpy().astype(np.float64), ref_lse)
