"""Pins for the fp64 oracle: closed forms, invariants, library special cases and
brute force. None of these retypes the oracle's formula; each is chosen so that a
plausible mistake (a dropped 1/sqrt(d), a transposed factor, a wrong GQA index,
a missing scale, a sign error in the merge) fails at least one of them, which
test_planted_mistakes_are_caught demonstrates on broken copies of the oracle."""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import lrkv_oracle as orc

HERE = os.path.dirname(os.path.abspath(__file__))


def rand_case(seed, B=2, Hq=4, Hkv=2, d=8, r=4, L=9, ragged=True, quant=False):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, Hq, d))
    ZK = rng.standard_normal((B, Hkv, L, r))
    ZV = rng.standard_normal((B, Hkv, L, r))
    BK = rng.standard_normal((Hkv, r, d))
    BV = rng.standard_normal((Hkv, r, d))
    seqlens = rng.integers(1, L + 1, size=B) if ragged else np.full(B, L)
    SK = rng.uniform(0.5, 2.0, (B, Hkv, L)) if quant else None
    SV = rng.uniform(0.5, 2.0, (B, Hkv, L)) if quant else None
    return q, ZK, ZV, BK, BV, seqlens, SK, SV


# ---- pin checks, parameterised by the attention implementation under test ----------


def check_identity_factors_equal_sdpa(attn):
    """r = d and B = I: the latents are the keys/values, so the result must equal
    torch's scaled_dot_product_attention (fp64, CPU) with KV heads repeated G times."""
    rng = np.random.default_rng(5)
    B, Hq, Hkv, d, L = 2, 6, 3, 8, 7
    q = rng.standard_normal((B, Hq, d))
    ZK = rng.standard_normal((B, Hkv, L, d))
    ZV = rng.standard_normal((B, Hkv, L, d))
    eye = np.stack([np.eye(d)] * Hkv)
    seqlens = np.full(B, L)
    out, lse = attn(q, ZK, ZV, eye, eye, seqlens)
    G = Hq // Hkv
    tq = torch.from_numpy(q)[:, :, None, :]
    tk = torch.from_numpy(ZK).repeat_interleave(G, dim=1)
    tv = torch.from_numpy(ZV).repeat_interleave(G, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv)[:, :, 0, :].numpy()
    s = torch.einsum("bhd,bhld->bhl", torch.from_numpy(q), tk) / math.sqrt(d)
    ref_lse = torch.logsumexp(s, dim=-1).numpy()
    return np.allclose(out, ref, atol=1e-12, rtol=0) and np.allclose(lse, ref_lse, atol=1e-12)


def check_zero_query_gives_mean(attn):
    """q = 0: every score is 0, so the output is the plain mean of the rebuilt values
    over the valid positions, and lse = ln L_b."""
    q, ZK, ZV, BK, BV, seqlens, _, _ = rand_case(11)
    q = np.zeros_like(q)
    out, lse = attn(q, ZK, ZV, BK, BV, seqlens)
    G = q.shape[1] // ZK.shape[1]
    ok = True
    for b in range(q.shape[0]):
        Lb = seqlens[b]
        for h in range(q.shape[1]):
            g = h // G
            mean_v = ZV[b, g, :Lb].mean(axis=0) @ BV[g]
            ok &= np.allclose(out[b, h], mean_v, atol=1e-12)
            ok &= abs(lse[b, h] - math.log(Lb)) < 1e-12
    return bool(ok)


def check_single_and_two_token_closed_forms(attn):
    """L = 1: out = V_0 exactly. L = 2: out = sigma(s0 - s1) V_0 + sigma(s1 - s0) V_1."""
    rng = np.random.default_rng(3)
    d, r = 6, 3
    q = rng.standard_normal((1, 1, d))
    ZK = rng.standard_normal((1, 1, 2, r))
    ZV = rng.standard_normal((1, 1, 2, r))
    BK = rng.standard_normal((1, r, d))
    BV = rng.standard_normal((1, r, d))
    out1, lse1 = attn(q, ZK, ZV, BK, BV, np.array([1]))
    v0 = ZV[0, 0, 0] @ BV[0]
    v1 = ZV[0, 0, 1] @ BV[0]
    k0 = ZK[0, 0, 0] @ BK[0]
    k1 = ZK[0, 0, 1] @ BK[0]
    s0 = k0 @ q[0, 0] / math.sqrt(d)
    s1 = k1 @ q[0, 0] / math.sqrt(d)
    ok = np.allclose(out1[0, 0], v0, atol=1e-13) and abs(lse1[0, 0] - s0) < 1e-13
    out2, lse2 = attn(q, ZK, ZV, BK, BV, np.array([2]))
    sig = 1.0 / (1.0 + math.exp(-(s0 - s1)))
    ok &= np.allclose(out2[0, 0], sig * v0 + (1 - sig) * v1, atol=1e-13)
    ok &= abs(lse2[0, 0] - (max(s0, s1) + math.log1p(math.exp(-abs(s0 - s1))))) < 1e-13
    return bool(ok)


def brute_force(q, ZK, ZV, BK, BV, seqlens, SK=None, SV=None):
    """Pure-Python loops, no numpy linear algebra (tiny shapes only)."""
    B, Hq, d = q.shape
    Hkv, r = ZK.shape[1], ZK.shape[3]
    G = Hq // Hkv
    out = np.zeros((B, Hq, d))
    lse = np.full((B, Hq), -np.inf)
    for b in range(B):
        for h in range(Hq):
            g = h // G
            Lb = int(seqlens[b])
            if Lb == 0:
                continue
            scores, vals = [], []
            for t in range(Lb):
                sk = 1.0 if SK is None else float(SK[b, g, t])
                sv = 1.0 if SV is None else float(SV[b, g, t])
                k = [sum(float(ZK[b, g, t, i]) * sk * float(BK[g, i, c]) for i in range(r))
                     for c in range(d)]
                v = [sum(float(ZV[b, g, t, i]) * sv * float(BV[g, i, c]) for i in range(r))
                     for c in range(d)]
                scores.append(sum(float(q[b, h, c]) * k[c] for c in range(d)) / math.sqrt(d))
                vals.append(v)
            m = max(scores)
            w = [math.exp(s - m) for s in scores]
            tot = sum(w)
            for c in range(d):
                out[b, h, c] = sum(w[t] * vals[t][c] for t in range(Lb)) / tot
            lse[b, h] = m + math.log(tot)
    return out, lse


def check_brute_force_tiny(attn):
    ok = True
    for seed in range(4):
        q, ZK, ZV, BK, BV, seqlens, SK, SV = rand_case(100 + seed, B=2, Hq=4, Hkv=2, d=4, r=3,
                                                        L=4, quant=(seed % 2 == 1))
        out, lse = attn(q, ZK, ZV, BK, BV, seqlens, SK, SV)
        ref, ref_lse = brute_force(q, ZK, ZV, BK, BV, seqlens, SK, SV)
        ok &= np.allclose(out, ref, atol=1e-12) and np.allclose(lse, ref_lse, atol=1e-12)
    return bool(ok)


def check_gqa_expansion(attn):
    """Repeating each KV head G times and running with G = 1 gives the same result."""
    q, ZK, ZV, BK, BV, seqlens, _, _ = rand_case(21, Hq=6, Hkv=2)
    out, lse = attn(q, ZK, ZV, BK, BV, seqlens)
    G = 3
    ZK2 = np.repeat(ZK, G, axis=1)
    ZV2 = np.repeat(ZV, G, axis=1)
    out2, lse2 = attn(q, ZK2, ZV2, np.repeat(BK, G, axis=0), np.repeat(BV, G, axis=0), seqlens)
    return np.allclose(out, out2, atol=1e-12) and np.allclose(lse, lse2, atol=1e-12)


def check_reassociation(attn):
    """(q B_K^T) Z_K^T and (p Z_V) B_V equal the rebuilt-K/V form (exact algebra)."""
    q, ZK, ZV, BK, BV, seqlens, SK, SV = rand_case(31, quant=True)
    out, lse = attn(q, ZK, ZV, BK, BV, seqlens, SK, SV)
    out2, lse2 = orc.decode_attention_reassociated(q, ZK, ZV, BK, BV, seqlens, SK, SV)
    return np.allclose(out, out2, atol=1e-12) and np.allclose(lse, lse2, atol=1e-12)


def check_golden(attn):
    with open(os.path.join(HERE, "golden", "hand_examples.json")) as f:
        cases = json.load(f)["cases"]
    ok = True
    for c in cases:
        nan = lambda a: np.array(a, dtype=np.float64)  # None -> nan
        q = nan(c["q"])
        ZK, ZV = nan(c["ZK"]), nan(c["ZV"])
        BK, BV = nan(c["BK"]), nan(c["BV"])
        SK = nan(c["ZK_scale"]) if "ZK_scale" in c else None
        SV = nan(c["ZV_scale"]) if "ZV_scale" in c else None
        seqlens = np.array(c["seqlens"])
        out, lse = attn(q, ZK, ZV, BK, BV, seqlens, SK, SV)
        exp_lse = np.array([[(-np.inf if v is None else v) for v in row] for row in c["lse"]])
        ok &= np.allclose(out, nan(c["out"]), atol=c["tol"], rtol=0)
        ok &= bool(np.all((np.isinf(exp_lse) & np.isinf(lse)) |
                          (np.abs(np.nan_to_num(lse - exp_lse, nan=1.0)) <= c["tol"])))
    return bool(ok)


PIN_CHECKS = [check_identity_factors_equal_sdpa, check_zero_query_gives_mean,
              check_single_and_two_token_closed_forms, check_brute_force_tiny,
              check_gqa_expansion, check_reassociation, check_golden]


def _oracle(q, ZK, ZV, BK, BV, seqlens, SK=None, SV=None):
    return orc.decode_attention(q, ZK, ZV, BK, BV, seqlens, SK, SV)


@pytest.mark.parametrize("check", PIN_CHECKS, ids=lambda f: f.__name__)
def test_oracle_pins(check):
    assert check(_oracle)


def test_score_shift_invariance():
    """Adding a constant to every score leaves the output unchanged (the softmax
    stabilisation must not change the result)."""
    q, ZK, ZV, BK, BV, seqlens, _, _ = rand_case(41)
    out, lse = orc.decode_attention(q, ZK, ZV, BK, BV, seqlens)
    for shift in (-50.0, 7.25, 300.0):
        out2, lse2 = orc.decode_attention(q, ZK, ZV, BK, BV, seqlens, score_shift=shift)
        assert np.allclose(out, out2, atol=1e-12)
        assert np.allclose(lse2 - lse, shift, atol=1e-9)


def test_split_merge_equals_unsplit():
    """Every split count from 1 to L_b (including splits past L_b that are empty)
    merges back to the unsplit result."""
    q, ZK, ZV, BK, BV, seqlens, SK, SV = rand_case(51, L=11, quant=True)
    ref, ref_lse = orc.decode_attention(q, ZK, ZV, BK, BV, seqlens, SK, SV)
    for chunk in range(1, 12):
        n_splits = -(-11 // chunk) + 1   # one always-empty trailing split
        o, l = orc.split_partials(q, ZK, ZV, BK, BV, seqlens, chunk, n_splits, SK, SV)
        out, lse = orc.merge_partials(o, l)
        assert np.allclose(out, ref, atol=1e-12)
        assert np.allclose(lse, ref_lse, atol=1e-12)


def test_merge_all_empty_row():
    o = np.zeros((1, 2, 3, 4))
    l = np.full((1, 2, 3), -np.inf)
    out, lse = orc.merge_partials(o, l)
    assert np.all(out == 0) and np.all(np.isneginf(lse))


# ---- stored formats -------------------------------------------------------------------


def test_bf16_decoder_matches_torch_all_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    mine = orc.bf16_bits_to_f64(bits)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(mine), nan)
    assert np.array_equal(mine[~nan], ref[~nan])


def test_bf16_encoder_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * 1e3,
        # exact ties: bf16 value + half an ulp, both parities of the kept lsb
        (np.arange(1, 2000, dtype=np.uint32) << 16 | 0x8000).view(np.float32),
        np.array([0.0, -0.0, 1e-40, -3e38, 3.4e38], dtype=np.float32)])
    mine = orc.f32_to_bf16_bits_rne(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(mine, ref)


def test_e4m3_decoder_matches_torch_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    mine = orc.e4m3_to_f64(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(mine), nan) and nan.sum() == 2
    assert np.array_equal(mine[~nan], ref[~nan])
    assert np.nanmax(mine) == 448.0


def test_e4m3_encoder_matches_torch_in_range():
    """torch's float32 -> float8_e4m3fn cast rounds to nearest even; it maps values
    above 464 to NaN, so it is compared only where both agree on finiteness."""
    vals = orc.e4m3_to_f64(np.arange(0x7F, dtype=np.uint8))
    mids = (vals[:-1] + vals[1:]) / 2            # exact ties
    rng = np.random.default_rng(1)
    x = np.concatenate([vals, -vals, mids, -mids, rng.uniform(-464, 464, 5000),
                        rng.standard_normal(5000) * 0.01]).astype(np.float32)
    mine = orc.f32_to_e4m3_rne_sat(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(mine, ref)


def test_e4m3_encoder_saturates():
    x = np.array([448.0, 449.0, 500.0, 1e9, -1e9, -449.0], dtype=np.float32)
    assert orc.f32_to_e4m3_rne_sat(x).tolist() == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE]
    assert orc.f32_to_e4m3_rne_sat(np.array([np.nan], np.float32))[0] == 0x7F


def test_int8_quantiser_properties():
    rng = np.random.default_rng(2)
    for _ in range(200):
        z = (rng.standard_normal(32) * rng.uniform(0.01, 100)).astype(np.float32)
        c, s = orc.quantise_int8_row(z)
        assert c.dtype == np.int8 and np.all(np.abs(c.astype(int)) <= 127)
        assert abs(int(c[np.argmax(np.abs(z))])) == 127
        err = np.abs(z.astype(np.float64) - c.astype(np.float64) * float(s))
        assert np.all(err <= 0.5 * float(s) * (1 + 1e-6))
    # ties go to even: absmax 127 gives scale exactly 1
    c, s = orc.quantise_int8_row(np.array([127.0, 2.5, 3.5, -2.5, -0.5], np.float32))
    assert s == 1.0 and c.tolist() == [127, 2, 4, -2, 0]
    c, s = orc.quantise_int8_row(np.zeros(8, np.float32))
    assert s == 1.0 and not c.any()


def test_e4m3_quantiser_properties():
    rng = np.random.default_rng(3)
    for _ in range(50):
        z = (rng.standard_normal(32) * rng.uniform(0.01, 100)).astype(np.float32)
        c, s = orc.quantise_e4m3_row(z)
        v = orc.e4m3_to_f64(c) * float(s)
        assert abs(orc.e4m3_to_f64(c[np.argmax(np.abs(z))])) == 448.0
        # relative rounding error of e4m3 is at most 2^-4 for normal values
        big = np.abs(z) > 2.0 ** -6 * float(s) * 2
        assert np.all(np.abs(v[big] - z[big]) <= np.abs(z[big]) * 2.0 ** -4 * (1 + 1e-6))


def test_append_semantics():
    rng = np.random.default_rng(4)
    B, Hkv, L, r = 3, 2, 5, 8
    for lat in ("f32", "bf16", "i8", "e4m3"):
        dt = {"f32": np.float32, "bf16": np.uint16, "i8": np.int8, "e4m3": np.uint8}[lat]
        ZK = np.zeros((B, Hkv, L, r), dt)
        ZV = np.zeros((B, Hkv, L, r), dt)
        quant = lat in ("i8", "e4m3")
        SK = np.zeros((B, Hkv, L), np.float32) if quant else None
        SV = np.zeros((B, Hkv, L), np.float32) if quant else None
        seqlens = np.array([0, 3, 5], np.int32)      # the last row is full
        zk = rng.standard_normal((B, Hkv, r)).astype(np.float32)
        zv = rng.standard_normal((B, Hkv, r)).astype(np.float32)
        ZK2, ZV2, SK2, SV2, sl2, status = orc.append(ZK, ZV, SK, SV, seqlens, zk, zv, lat)
        assert sl2.tolist() == [1, 4, 5] and status == orc.STATUS_APPEND_FULL
        assert np.array_equal(ZK2[2], ZK[2])
        for b, slot in ((0, 0), (1, 3)):
            dec_k = orc.decode_stored(ZK2[b, :, slot], lat)
            if quant:
                dec_k = dec_k * SK2[b, :, slot, None]
            tol = {"f32": 0, "bf16": 2 ** -8, "i8": 1 / 127, "e4m3": 2 ** -4}[lat]
            assert np.all(np.abs(dec_k - zk[b]) <= tol * np.abs(zk[b]).max(axis=-1, keepdims=True)
                          + 1e-12)
            # untouched neighbouring slots
            assert not ZK2[b, :, slot + 1:].any()


# ---- planted mistakes: each broken copy must fail at least one pin ---------------------


def _mutant(kind):
    def attn(q, ZK, ZV, BK, BV, seqlens, SK=None, SV=None):
        q = np.asarray(q, np.float64)
        B, Hq, d = q.shape
        Hkv = ZK.shape[1]
        G = Hq // Hkv
        out = np.zeros((B, Hq, d))
        lse = np.full((B, Hq), -np.inf)
        for b in range(B):
            Lb = int(seqlens[b]) + (1 if kind == "off-by-one-length" else 0)
            Lb = min(Lb, ZK.shape[2])
            for h in range(Hq):
                g = (h % Hkv) if kind == "gqa-modulo" else h // G
                Zk = np.asarray(ZK[b, g, :Lb], np.float64)
                Zv = np.asarray((ZK if kind == "v-from-zk" else ZV)[b, g, :Lb], np.float64)
                if SK is not None and kind != "drop-scale":
                    Zk = Zk * SK[b, g, :Lb, None]
                if SV is not None and kind != "drop-scale":
                    Zv = Zv * SV[b, g, :Lb, None]
                K = Zk @ (BV[g] if kind == "bk-bv-swapped" else BK[g])
                V = Zv @ BV[g]
                scale = 1.0 if kind == "no-sqrt-d" else 1.0 / math.sqrt(d)
                s = (K @ q[b, h]) * scale
                if Lb == 0:
                    continue
                m = s.max()
                e = np.exp(s - m)
                l = e.sum()
                out[b, h] = (e / (l if kind != "unnormalised" else 1.0)) @ V
                lse[b, h] = (m + math.log(l)) if kind != "lse-no-max" else math.log(l)
        return out, lse
    return attn


@pytest.mark.parametrize("kind", ["off-by-one-length", "gqa-modulo", "v-from-zk", "drop-scale",
                                  "bk-bv-swapped", "no-sqrt-d", "unnormalised", "lse-no-max"])
def test_planted_mistakes_are_caught(kind):
    broken = _mutant(kind)
    failures = []
    for check in PIN_CHECKS:
        try:
            ok = check(broken)
        except Exception:
            ok = False
        if not ok:
            failures.append(check.__name__)
    assert failures, f"no pin caught the planted mistake {kind!r}"
