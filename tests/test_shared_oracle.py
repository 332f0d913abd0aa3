"""Pins of the oracle's cross-head shared latent (one latent per token for every KV
head and one decompression matrix for all heads; "AttentionPack", Metodologia 2.A).

- a block-diagonal decompression over per-head latents placed side by side is the
  per-head low-rank cache: equal to decode_attention;
- identity decompression (R = H d, D = I) is plain attention over the stored rows:
  equal to torch SDPA with KV heads repeated;
- a token-by-token pure-Python loop agrees, quantised scales included;
- the planted mistakes of reading the wrong head's column block, or of the
  transposed (dimension-major) concatenation, fail a pin.
"""
import math

import numpy as np
import torch

from oracle import lrkv_oracle as orc


def test_block_diagonal_equals_per_head_cache():
    rng = np.random.default_rng(1)
    B, Hq, Hkv, d, r, L = 2, 6, 3, 4, 2, 7
    q = rng.standard_normal((B, Hq, d))
    ZKh = rng.standard_normal((B, Hkv, L, r))
    ZVh = rng.standard_normal((B, Hkv, L, r))
    BK = rng.standard_normal((Hkv, r, d))
    BV = rng.standard_normal((Hkv, r, d))
    seq = np.array([L, 4])
    # shared form: latent [B][L][Hkv r], decompression block-diagonal [Hkv r][Hkv d]
    ZK = ZKh.transpose(0, 2, 1, 3).reshape(B, L, Hkv * r)
    ZV = ZVh.transpose(0, 2, 1, 3).reshape(B, L, Hkv * r)
    DK = np.zeros((Hkv * r, Hkv * d))
    DV = np.zeros((Hkv * r, Hkv * d))
    for g in range(Hkv):
        DK[g * r:(g + 1) * r, g * d:(g + 1) * d] = BK[g]
        DV[g * r:(g + 1) * r, g * d:(g + 1) * d] = BV[g]
    got = orc.decode_attention_shared(q, ZK, ZV, DK, DV, seq, Hkv)
    ref = orc.decode_attention(q, ZKh, ZVh, BK, BV, seq)
    np.testing.assert_allclose(got[0], ref[0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(got[1], ref[1], rtol=0, atol=1e-12)


def test_identity_decompression_equals_sdpa():
    rng = np.random.default_rng(2)
    B, Hq, Hkv, d, L = 2, 4, 2, 8, 6
    q = rng.standard_normal((B, Hq, d))
    ZK = rng.standard_normal((B, L, Hkv * d))
    ZV = rng.standard_normal((B, L, Hkv * d))
    eye = np.eye(Hkv * d)
    out, lse = orc.decode_attention_shared(q, ZK, ZV, eye, eye, np.full(B, L), Hkv)
    K = torch.from_numpy(ZK).reshape(B, L, Hkv, d).permute(0, 2, 1, 3).repeat_interleave(2, dim=1)
    V = torch.from_numpy(ZV).reshape(B, L, Hkv, d).permute(0, 2, 1, 3).repeat_interleave(2, dim=1)
    tq = torch.from_numpy(q)[:, :, None, :]
    ref = torch.nn.functional.scaled_dot_product_attention(tq, K, V)[:, :, 0, :].numpy()
    ref_lse = torch.logsumexp(torch.einsum("bhd,bhld->bhl", torch.from_numpy(q), K) / math.sqrt(d),
                              dim=-1).numpy()
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


def _loop(q, ZK, ZV, DK, DV, seq, Hkv, SK=None, SV=None, col=lambda g, c, d, H: g * d + c):
    B, Hq, d = q.shape
    R = ZK.shape[2]
    G = Hq // Hkv
    out = np.zeros((B, Hq, d))
    lse = np.full((B, Hq), -np.inf)
    for b in range(B):
        L = int(seq[b])
        for h in range(Hq):
            g = h // G
            scores, vals = [], []
            for t in range(L):
                sk = 1.0 if SK is None else float(SK[b, t])
                sv = 1.0 if SV is None else float(SV[b, t])
                k = [sum(float(ZK[b, t, j]) * sk * float(DK[j, col(g, c, d, Hkv)]) for j in range(R))
                     for c in range(d)]
                v = [sum(float(ZV[b, t, j]) * sv * float(DV[j, col(g, c, d, Hkv)]) for j in range(R))
                     for c in range(d)]
                scores.append(sum(float(q[b, h, c]) * k[c] for c in range(d)) / math.sqrt(d))
                vals.append(v)
            mx = max(scores)
            w = [math.exp(x - mx) for x in scores]
            tot = sum(w)
            for c in range(d):
                out[b, h, c] = sum(w[t] * vals[t][c] for t in range(L)) / tot
            lse[b, h] = mx + math.log(tot)
    return out, lse


def _case(seed, quant=False):
    rng = np.random.default_rng(seed)
    B, Hq, Hkv, d, R, L = 2, 4, 2, 3, 5, 6
    q = rng.standard_normal((B, Hq, d))
    ZK = rng.standard_normal((B, L, R))
    ZV = rng.standard_normal((B, L, R))
    DK = rng.standard_normal((R, Hkv * d))
    DV = rng.standard_normal((R, Hkv * d))
    SK = rng.uniform(0.5, 2.0, (B, L)) if quant else None
    SV = rng.uniform(0.5, 2.0, (B, L)) if quant else None
    return q, ZK, ZV, DK, DV, np.array([L, 3]), Hkv, SK, SV


def test_pure_python_loop_agrees():
    for quant in (False, True):
        q, ZK, ZV, DK, DV, seq, Hkv, SK, SV = _case(3 + quant, quant)
        got = orc.decode_attention_shared(q, ZK, ZV, DK, DV, seq, Hkv, SK, SV)
        ref = _loop(q, ZK, ZV, DK, DV, seq, Hkv, SK, SV)
        np.testing.assert_allclose(got[0], ref[0], rtol=0, atol=1e-12)
        np.testing.assert_allclose(got[1], ref[1], rtol=0, atol=1e-12)


def test_planted_mistakes_fail_the_loop_pin():
    q, ZK, ZV, DK, DV, seq, Hkv, _, _ = _case(5)
    got = orc.decode_attention_shared(q, ZK, ZV, DK, DV, seq, Hkv)
    other_head = _loop(q, ZK, ZV, DK, DV, seq, Hkv, col=lambda g, c, d, H: ((g + 1) % H) * d + c)
    dim_major = _loop(q, ZK, ZV, DK, DV, seq, Hkv, col=lambda g, c, d, H: c * H + g)
    for bad in (other_head, dim_major):
        assert not np.allclose(got[0], bad[0], atol=1e-6)
