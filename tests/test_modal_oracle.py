"""Pins of the oracle's modality-separated factors (visual rows rebuilt with one factor
set, text rows with another; "AttentionPack", Metodologia 2.A, modal separation).

- two identical sets give the single-set result, whatever the boundary;
- a boundary at or past the row length uses the visual set only, which equals the
  single-set result with that set;
- identity-like sets reduce to torch SDPA over explicitly rebuilt keys and values;
- a pure-Python loop that picks the set token by token agrees on tiny shapes with
  the boundary inside the rows, quantised scales included;
- the planted mistakes of an off-by-one boundary and of swapped sets fail the loop pin.
"""
import math

import numpy as np
import pytest
import torch

from oracle import lrkv_oracle as orc


def _case(seed, B=3, Hq=4, Hkv=2, d=4, r=3, L=9, quant=False):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, Hq, d))
    ZK = rng.standard_normal((B, Hkv, L, r))
    ZV = rng.standard_normal((B, Hkv, L, r))
    BK = rng.standard_normal((2, Hkv, r, d))
    BV = rng.standard_normal((2, Hkv, r, d))
    seqlens = np.array([L, 2, 6][:B])
    SK = rng.uniform(0.5, 2.0, (B, Hkv, L)) if quant else None
    SV = rng.uniform(0.5, 2.0, (B, Hkv, L)) if quant else None
    return q, ZK, ZV, BK, BV, seqlens, SK, SV


def _loop(q, ZK, ZV, BK, BV, seqlens, P, SK=None, SV=None, boundary=lambda t, P: t < P):
    """Token by token: key/value of token t rebuilt with set 0 if boundary(t, P)."""
    B, Hq, d = q.shape
    Hkv, r = ZK.shape[1], ZK.shape[3]
    G = Hq // Hkv
    out = np.zeros((B, Hq, d))
    lse = np.full((B, Hq), -np.inf)
    for b in range(B):
        for h in range(Hq):
            g = h // G
            Lb = int(seqlens[b])
            scores, vals = [], []
            for t in range(Lb):
                m = 0 if boundary(t, P) else 1
                sk = 1.0 if SK is None else float(SK[b, g, t])
                sv = 1.0 if SV is None else float(SV[b, g, t])
                k = [sum(float(ZK[b, g, t, i]) * sk * float(BK[m, g, i, c]) for i in range(r))
                     for c in range(d)]
                v = [sum(float(ZV[b, g, t, i]) * sv * float(BV[m, g, i, c]) for i in range(r))
                     for c in range(d)]
                scores.append(sum(float(q[b, h, c]) * k[c] for c in range(d)) / math.sqrt(d))
                vals.append(v)
            if not scores:
                continue
            mx = max(scores)
            w = [math.exp(s - mx) for s in scores]
            tot = sum(w)
            for c in range(d):
                out[b, h, c] = sum(w[t] * vals[t][c] for t in range(Lb)) / tot
            lse[b, h] = mx + math.log(tot)
    return out, lse


@pytest.mark.parametrize("P", [1, 3, 5, 8, 9, 40])
def test_identical_sets_equal_single_set(P):
    q, ZK, ZV, BK, BV, seq, _, _ = _case(1)
    BK2, BV2 = np.stack([BK[1], BK[1]]), np.stack([BV[0], BV[0]])
    got = orc.decode_attention(q, ZK, ZV, BK2, BV2, seq, n_visual=P)
    ref = orc.decode_attention(q, ZK, ZV, BK[1], BV[0], seq)
    np.testing.assert_allclose(got[0], ref[0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(got[1], ref[1], rtol=0, atol=1e-12)


def test_boundary_past_length_uses_visual_set_only():
    q, ZK, ZV, BK, BV, seq, _, _ = _case(2)
    got = orc.decode_attention(q, ZK, ZV, BK, BV, seq, n_visual=int(seq.max()))
    ref = orc.decode_attention(q, ZK, ZV, BK[0], BV[0], seq)
    np.testing.assert_array_equal(got[0], ref[0])
    np.testing.assert_array_equal(got[1], ref[1])


def test_matches_sdpa_over_explicitly_rebuilt_rows():
    """Rebuild every row with its own set by hand (torch), then torch SDPA."""
    q, ZK, ZV, BK, BV, _, _, _ = _case(3, B=2, Hq=4, Hkv=2, d=8, r=5, L=7)
    P, L = 4, 7
    seq = np.full(2, L)
    out, lse = orc.decode_attention(q, ZK, ZV, BK, BV, seq, n_visual=P)
    tz_k, tz_v = torch.from_numpy(ZK), torch.from_numpy(ZV)
    K = torch.cat([torch.einsum("bgtr,grd->bgtd", tz_k[:, :, :P], torch.from_numpy(BK[0])),
                   torch.einsum("bgtr,grd->bgtd", tz_k[:, :, P:], torch.from_numpy(BK[1]))], dim=2)
    V = torch.cat([torch.einsum("bgtr,grd->bgtd", tz_v[:, :, :P], torch.from_numpy(BV[0])),
                   torch.einsum("bgtr,grd->bgtd", tz_v[:, :, P:], torch.from_numpy(BV[1]))], dim=2)
    G = 2
    K, V = K.repeat_interleave(G, dim=1), V.repeat_interleave(G, dim=1)
    tq = torch.from_numpy(q)[:, :, None, :]
    ref = torch.nn.functional.scaled_dot_product_attention(tq, K, V)[:, :, 0, :].numpy()
    ref_lse = torch.logsumexp(torch.einsum("bhd,bhld->bhl", torch.from_numpy(q), K) / math.sqrt(8),
                              dim=-1).numpy()
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


@pytest.mark.parametrize("quant", [False, True])
@pytest.mark.parametrize("P", [1, 4, 6])
def test_pure_python_loop_agrees(P, quant):
    q, ZK, ZV, BK, BV, seq, SK, SV = _case(10 + P, quant=quant)
    got = orc.decode_attention(q, ZK, ZV, BK, BV, seq, SK, SV, n_visual=P)
    ref = _loop(q, ZK, ZV, BK, BV, seq, P, SK, SV)
    np.testing.assert_allclose(got[0], ref[0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(got[1], ref[1], rtol=0, atol=1e-12)


def test_planted_mistakes_fail_the_loop_pin():
    q, ZK, ZV, BK, BV, seq, _, _ = _case(20)
    P = 4
    got = orc.decode_attention(q, ZK, ZV, BK, BV, seq, n_visual=P)
    off_by_one = _loop(q, ZK, ZV, BK, BV, seq, P, boundary=lambda t, P: t <= P)
    swapped = _loop(q, ZK, ZV, BK[::-1], BV[::-1], seq, P)
    for bad in (off_by_one, swapped):
        assert not np.allclose(got[0], bad[0], atol=1e-6)
