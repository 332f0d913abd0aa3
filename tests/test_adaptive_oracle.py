"""Pins of the oracle's attention-aware partial decompression (tokens below the
importance threshold rebuilt from the leading r_low rank components; the attention
mass tracked with a moving average; "AttentionPack", Metodologia 2.B).

- every token important (tau = -inf) or r_low = r: plain decode attention, and the
  mass of a row sums to G (the G heads' softmax weights);
- no token important (tau = +inf): plain decode attention over latents and factors
  truncated to their first r_low components (an independent path);
- the mass equals torch softmax weights summed over the group's heads;
- the moving average has its closed form (beta = 1 keeps, beta = 0 replaces) and
  positions past the length are untouched;
- a token-by-token pure-Python loop agrees with mixed importance, quantised scales
  and modality-separated factors;
- planted mistakes (inverted threshold, swapped moving-average weights) fail a pin.
"""
import math

import numpy as np
import pytest
import torch

from oracle import lrkv_oracle as orc


def _case(seed, B=2, Hq=4, Hkv=2, d=4, r=6, L=9, quant=False, sets=1):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, Hq, d))
    ZK = rng.standard_normal((B, Hkv, L, r))
    ZV = rng.standard_normal((B, Hkv, L, r))
    fshape = (Hkv, r, d) if sets == 1 else (2, Hkv, r, d)
    BK = rng.standard_normal(fshape)
    BV = rng.standard_normal(fshape)
    seqlens = np.array([L, 5][:B])
    imp = rng.uniform(0.0, 1.0, (B, Hkv, L)).astype(np.float32)
    SK = rng.uniform(0.5, 2.0, (B, Hkv, L)) if quant else None
    SV = rng.uniform(0.5, 2.0, (B, Hkv, L)) if quant else None
    return q, ZK, ZV, BK, BV, seqlens, imp, SK, SV


def test_all_important_is_plain_attention_and_mass_sums_to_group():
    q, ZK, ZV, BK, BV, seq, imp, _, _ = _case(1)
    out, lse, mass, _ = orc.decode_attention_adaptive(q, ZK, ZV, BK, BV, seq, imp, -np.inf, 2, 0.5)
    ref, ref_lse = orc.decode_attention(q, ZK, ZV, BK, BV, seq)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)
    G = q.shape[1] // ZK.shape[1]
    for b, L in enumerate(seq):
        np.testing.assert_allclose(mass[b, :, :L].sum(axis=1), G, rtol=0, atol=1e-12)
        assert np.all(mass[b, :, L:] == 0)
    full, *_ = orc.decode_attention_adaptive(q, ZK, ZV, BK, BV, seq, imp, 0.5, ZK.shape[3], 0.5)
    np.testing.assert_allclose(full, ref, rtol=0, atol=1e-12)


def test_none_important_equals_truncated_factors():
    q, ZK, ZV, BK, BV, seq, imp, _, _ = _case(2)
    rl = 2
    out, lse, _, _ = orc.decode_attention_adaptive(q, ZK, ZV, BK, BV, seq, imp, np.inf, rl, 0.5)
    ref, ref_lse = orc.decode_attention(q, ZK[..., :rl], ZV[..., :rl], BK[:, :rl], BV[:, :rl], seq)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


def test_mass_matches_torch_softmax_summed_over_group():
    q, ZK, ZV, BK, BV, seq, imp, _, _ = _case(3)
    tau, rl = 0.5, 3
    _, _, mass, _ = orc.decode_attention_adaptive(q, ZK, ZV, BK, BV, seq, imp, tau, rl, 0.5)
    B, Hq, d = q.shape
    Hkv = ZK.shape[1]
    G = Hq // Hkv
    for b in range(B):
        L = int(seq[b])
        for g in range(Hkv):
            zk = torch.from_numpy(ZK[b, g, :L].copy())
            low = torch.from_numpy(imp[b, g, :L] < tau)
            zk[low, rl:] = 0
            K = zk @ torch.from_numpy(BK[g])
            s = torch.from_numpy(q[b, g * G:(g + 1) * G]) @ K.T / math.sqrt(d)
            want = torch.softmax(s, dim=-1).sum(dim=0).numpy()
            np.testing.assert_allclose(mass[b, g, :L], want, rtol=0, atol=1e-12)


def test_moving_average_closed_forms():
    q, ZK, ZV, BK, BV, seq, imp, _, _ = _case(4)
    _, _, mass, keep = orc.decode_attention_adaptive(q, ZK, ZV, BK, BV, seq, imp, 0.4, 2, 1.0)
    np.testing.assert_array_equal(keep, imp.astype(np.float64))
    _, _, mass0, repl = orc.decode_attention_adaptive(q, ZK, ZV, BK, BV, seq, imp, 0.4, 2, 0.0)
    for b, L in enumerate(seq):
        np.testing.assert_array_equal(repl[b, :, :L], mass0[b, :, :L])
        np.testing.assert_array_equal(repl[b, :, L:], imp[b, :, L:].astype(np.float64))
    _, _, m, half = orc.decode_attention_adaptive(q, ZK, ZV, BK, BV, seq, imp, 0.4, 2, 0.25)
    L = int(seq[0])
    np.testing.assert_allclose(half[0, :, :L], 0.25 * imp[0, :, :L] + 0.75 * m[0, :, :L],
                               rtol=0, atol=1e-15)


def _loop(q, ZK, ZV, BK, BV, seq, imp, tau, rl, beta, SK=None, SV=None, n_visual=0,
          important=lambda v, tau: v >= tau, ema=lambda old, m, beta: beta * old + (1 - beta) * m):
    B, Hq, d = q.shape
    Hkv, r = ZK.shape[1], ZK.shape[3]
    G = Hq // Hkv
    out = np.zeros((B, Hq, d))
    lse = np.full((B, Hq), -np.inf)
    new = np.array(imp, np.float64)
    for b in range(B):
        L = int(seq[b])
        for g in range(Hkv):
            mass = [0.0] * L
            for h in range(g * G, (g + 1) * G):
                scores, vals = [], []
                for t in range(L):
                    rank = r if important(float(imp[b, g, t]), tau) else rl
                    m = 0 if (n_visual == 0 or t < n_visual) else 1
                    fk = BK[m][g] if n_visual else BK[g]
                    fv = BV[m][g] if n_visual else BV[g]
                    sk = 1.0 if SK is None else float(SK[b, g, t])
                    sv = 1.0 if SV is None else float(SV[b, g, t])
                    k = [sum(float(ZK[b, g, t, j]) * sk * float(fk[j, c]) for j in range(rank))
                         for c in range(d)]
                    v = [sum(float(ZV[b, g, t, j]) * sv * float(fv[j, c]) for j in range(rank))
                         for c in range(d)]
                    scores.append(sum(float(q[b, h, c]) * k[c] for c in range(d)) / math.sqrt(d))
                    vals.append(v)
                mx = max(scores)
                w = [math.exp(x - mx) for x in scores]
                tot = sum(w)
                for c in range(d):
                    out[b, h, c] = sum(w[t] * vals[t][c] for t in range(L)) / tot
                lse[b, h] = mx + math.log(tot)
                for t in range(L):
                    mass[t] += w[t] / tot
            for t in range(L):
                new[b, g, t] = ema(float(imp[b, g, t]), mass[t], beta)
    return out, lse, new


@pytest.mark.parametrize("quant,sets", [(False, 1), (True, 1), (False, 2)])
def test_pure_python_loop_agrees(quant, sets):
    q, ZK, ZV, BK, BV, seq, imp, SK, SV = _case(10 + 2 * quant + sets, quant=quant, sets=sets)
    nv = 4 if sets == 2 else 0
    got = orc.decode_attention_adaptive(q, ZK, ZV, BK, BV, seq, imp, 0.45, 2, 0.7, SK, SV,
                                        n_visual=nv)
    ref = _loop(q, ZK, ZV, BK, BV, seq, imp, 0.45, 2, 0.7, SK, SV, n_visual=nv)
    np.testing.assert_allclose(got[0], ref[0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(got[1], ref[1], rtol=0, atol=1e-12)
    np.testing.assert_allclose(got[3], ref[2], rtol=0, atol=1e-12)


def test_planted_mistakes_fail_the_loop_pin():
    q, ZK, ZV, BK, BV, seq, imp, _, _ = _case(30)
    got = orc.decode_attention_adaptive(q, ZK, ZV, BK, BV, seq, imp, 0.5, 2, 0.7)
    inverted = _loop(q, ZK, ZV, BK, BV, seq, imp, 0.5, 2, 0.7, important=lambda v, tau: v < tau)
    swapped = _loop(q, ZK, ZV, BK, BV, seq, imp, 0.5, 2, 0.7,
                    ema=lambda old, m, beta: (1 - beta) * old + beta * m)
    assert not np.allclose(got[0], inverted[0], atol=1e-6)
    assert not np.allclose(got[3], swapped[2], atol=1e-6)


def test_inputs_are_left_as_given():
    q, ZK, ZV, BK, BV, seq, imp, _, _ = _case(40)
    keep = [a.copy() for a in (q, ZK, ZV, BK, BV, imp)]
    orc.decode_attention_adaptive(q, ZK, ZV, BK, BV, seq, imp, 0.5, 2, 0.7)
    for a, b in zip((q, ZK, ZV, BK, BV, imp), keep):
        np.testing.assert_array_equal(a, b)
