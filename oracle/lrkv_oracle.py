"""fp64 CPU oracle for single-token decode attention over a per-head low-rank KV cache.

TEST INFRASTRUCTURE. Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline
and reference legs may import or call this module. It shares no code with the CUDA
path and imports nothing from the rank_kv_cache_head_b200 package. It is plain,
slow and meant to be checked by eye against the definitions below.

What is computed, and where it comes from:

* Per-head low-rank cache. Each KV head g keeps its own compact latent and an
  up-projection factor: W_K,g = A_K,g B_K,g with rank r much smaller than the full
  rank ("WSVD: Weighted Low-Rank Approximation for Fast and Efficient Execution of
  Low-Precision Vision-Language Models", §2.A, per-head SVD). The cached latent of a
  token is Z = x A (computed upstream); the key/value rows are rebuilt as
  K_g = Z_K,g B_K,g and V_g = Z_V,g B_V,g.
* Attention over the rebuilt rows, with reconstruction, attention and Flash
  Decoding in one flow (same page, §2.C, kernel fusion). The result is ordinary
  softmax attention over the rebuilt K, V, so the oracle is that definition
  written out: s = K q / sqrt(d), p = softmax(s), out = p V, lse = log sum exp(s).
* Flash Decoding splits the sequence into chunks, each yielding a normalised
  partial o_s and its log-sum-exp lse_s; the merge is
  out = sum_s exp(lse_s - LSE) o_s with LSE = log sum_s exp(lse_s).
* Query head h reads KV head floor(h / G), G = H_q / H_kv (contiguous grouping).
* Quantised latents carry one fp32 scale per (batch, KV head, token); the
  dequantised latent is code * scale. int8 codes are symmetric in [-127, 127];
  e4m3 is OCP FP8 E4M3FN (bias 7, no infinities, max 448).

Readings where the pages are silent (each is listed in the design notes too):
score scale 1/sqrt(d_head); no positional rotation applied to the rebuilt keys;
append precedes attend, so positions 0..L_b-1 are attended; a row with L_b = 0
gives out = 0 and lse = -inf; an empty split contributes nothing.

Parity pins: every function here is checked in tests/test_oracle.py against closed
forms, invariants, library routines (torch SDPA, torch's float8 and bf16 casts)
and brute force on tiny shapes. Absolute accuracy on a real model is parity
unpinned (no weights or datasets are available).
"""
from __future__ import annotations

import math

import numpy as np

# --------------------------------------------------------------------------------------
# Stored-format decoders and encoders (bit level, no library casts)
# --------------------------------------------------------------------------------------


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns (uint16) -> float64. bf16 is the top half of an fp32."""
    u32 = bits.astype(np.uint32) << np.uint32(16)
    return u32.view(np.float32).astype(np.float64)


def f32_to_bf16_bits_rne(x: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bits, round to nearest, ties to even (NaN kept quiet)."""
    x = np.asarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    rounded = (u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    out = rounded.astype(np.uint16)
    nan = np.isnan(x)
    out[nan] = ((u[nan] >> np.uint64(16)) | np.uint64(0x40)).astype(np.uint16)
    return out


def _e4m3_value(code: int) -> float:
    """Value of one OCP FP8 E4M3FN code (sign 1, exponent 4 with bias 7, mantissa 3)."""
    sign = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return sign * (m / 8.0) * 2.0 ** (1 - 7)
    return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)


_E4M3_TABLE = np.array([_e4m3_value(c) for c in range(256)], dtype=np.float64)
# non-negative finite codes 0x00..0x7E in increasing value order
_E4M3_POS_VALUES = _E4M3_TABLE[:0x7F].copy()
E4M3_MAX = 448.0


def e4m3_to_f64(codes: np.ndarray) -> np.ndarray:
    return _E4M3_TABLE[np.asarray(codes, dtype=np.uint8)]


def f32_to_e4m3_rne_sat(x: np.ndarray) -> np.ndarray:
    """float32 -> e4m3 codes: nearest representable value, ties to the even code,
    magnitudes above 448 saturate to 448 (the satfinite rule), NaN -> 0x7F."""
    x = np.asarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint8)
    flat_x = x.reshape(-1)
    flat_o = out.reshape(-1)
    for i, v in enumerate(flat_x):
        if math.isnan(v):
            flat_o[i] = 0x7F
            continue
        sign = 0x80 if (v < 0 or (v == 0 and math.copysign(1.0, v) < 0)) else 0
        a = abs(v)
        if a >= E4M3_MAX:
            flat_o[i] = sign | 0x7E
            continue
        hi = int(np.searchsorted(_E4M3_POS_VALUES, a, side="left"))  # first value >= a
        if _E4M3_POS_VALUES[hi] == a:
            code = hi
        else:
            lo = hi - 1
            dlo = a - _E4M3_POS_VALUES[lo]
            dhi = _E4M3_POS_VALUES[hi] - a
            if dlo < dhi:
                code = lo
            elif dhi < dlo:
                code = hi
            else:
                code = lo if lo % 2 == 0 else hi
        flat_o[i] = sign | code
    return out


def decode_stored(x: np.ndarray, dtype: str) -> np.ndarray:
    """Stored latent / io values -> float64 (exact for every supported format)."""
    if dtype == "f32":
        return np.asarray(x, dtype=np.float32).astype(np.float64)
    if dtype == "bf16":
        return bf16_bits_to_f64(np.asarray(x, dtype=np.uint16))
    if dtype == "i8":
        return np.asarray(x, dtype=np.int8).astype(np.float64)
    if dtype == "e4m3":
        return e4m3_to_f64(x)
    raise ValueError(dtype)


# --------------------------------------------------------------------------------------
# Decode attention (the definition)
# --------------------------------------------------------------------------------------


def dequantise(Z: np.ndarray, scale) -> np.ndarray:
    """code * per-token scale (scale None for unquantised latents)."""
    if scale is None:
        return Z
    return Z * scale[..., None]


def decode_attention(q, ZK, ZV, BK, BV, seqlens, ZK_scale=None, ZV_scale=None,
                     score_shift: float = 0.0, pairs=None, n_visual: int = 0):
    """Single-token decode attention over a per-head low-rank cache, in float64.

    q [B][Hq][d]; ZK, ZV [B][Hkv][L_cap][r] (decoded codes); scales [B][Hkv][L_cap]
    or None; BK, BV [Hkv][r][d]; seqlens [B]. Returns out [B][Hq][d], lse [B][Hq]
    (natural log). ``score_shift`` adds a constant to every score (used only to pin
    the softmax stabilisation). ``pairs`` restricts the work to some (b, h).

    Modality-separated factors ("AttentionPack", Metodologia 2.A: visual and text
    tokens are compressed separately because their distributions differ): with
    n_visual > 0, BK and BV are [2][Hkv][r][d]; positions t < n_visual of every row
    are rebuilt with the first (visual) set and positions t >= n_visual with the
    second (text) set. Reading: one boundary shared by every row, visual tokens first.
    """
    q = np.asarray(q, np.float64)
    B, Hq, d = q.shape
    Hkv = ZK.shape[1]
    G = Hq // Hkv
    out = np.zeros((B, Hq, d))
    lse = np.full((B, Hq), -np.inf)
    want = None if pairs is None else set(map(tuple, pairs))
    for b in range(B):
        Lb = int(seqlens[b])
        for g in range(Hkv):
            heads = [h for h in range(g * G, (g + 1) * G) if want is None or (b, h) in want]
            if not heads or Lb == 0:
                continue
            sk = None if ZK_scale is None else ZK_scale[b, g, :Lb]
            sv = None if ZV_scale is None else ZV_scale[b, g, :Lb]
            Zk = dequantise(np.asarray(ZK[b, g, :Lb, :], np.float64), sk)
            Zv = dequantise(np.asarray(ZV[b, g, :Lb, :], np.float64), sv)
            if n_visual > 0:
                P = min(n_visual, Lb)                    # visual rows, then text rows
                K = np.concatenate([Zk[:P] @ np.asarray(BK[0][g], np.float64),
                                    Zk[P:] @ np.asarray(BK[1][g], np.float64)])
                V = np.concatenate([Zv[:P] @ np.asarray(BV[0][g], np.float64),
                                    Zv[P:] @ np.asarray(BV[1][g], np.float64)])
            else:
                K = Zk @ np.asarray(BK[g], np.float64)   # Lb x d, rebuilt keys
                V = Zv @ np.asarray(BV[g], np.float64)   # Lb x d, rebuilt values
            for h in heads:
                s = (K @ q[b, h]) / math.sqrt(d) + score_shift
                m = s.max()
                e = np.exp(s - m)
                l = e.sum()
                out[b, h] = (e / l) @ V
                lse[b, h] = m + math.log(l)
    return out, lse


def decode_attention_adaptive(q, ZK, ZV, BK, BV, seqlens, importance, tau: float, r_low: int,
                              beta: float, ZK_scale=None, ZV_scale=None, n_visual: int = 0):
    """Attention-aware partial decompression ("AttentionPack", Metodologia 2.B): tokens
    whose tracked importance is high are rebuilt at the full rank, the others with the
    leading r_low rank components only (the factor rows are ordered by singular value,
    so a prefix is the best rank-r_low part); the accumulated attention is tracked with
    a moving average.

    Readings: importance is kept per (batch row, KV head, token) in ``importance``
    [B][Hkv][L_cap] (fp32 values); a token is important when importance >= tau (the
    comparison of the stored fp32 values); the reduced rank applies to both the key and
    the value row; a token's attention mass is its softmax weight summed over the G query
    heads of the group, and the moving average is imp <- beta * imp + (1 - beta) * mass
    for the attended positions (the others are left unchanged).

    Returns out [B][Hq][d], lse [B][Hq], mass [B][Hkv][L_cap] (0 past the length) and
    the updated importance [B][Hkv][L_cap] (float64)."""
    q = np.asarray(q, np.float64)
    B, Hq, d = q.shape
    Hkv, Lc, r = ZK.shape[1], ZK.shape[2], ZK.shape[3]
    G = Hq // Hkv
    imp = np.asarray(importance, np.float64)
    out = np.zeros((B, Hq, d))
    lse = np.full((B, Hq), -np.inf)
    mass = np.zeros((B, Hkv, Lc))
    for b in range(B):
        Lb = int(seqlens[b])
        if Lb == 0:
            continue
        for g in range(Hkv):
            sk = None if ZK_scale is None else ZK_scale[b, g, :Lb]
            sv = None if ZV_scale is None else ZV_scale[b, g, :Lb]
            # copies: the reduced-rank rows are edited below, the inputs stay as given
            Zk = np.array(dequantise(np.asarray(ZK[b, g, :Lb, :], np.float64), sk))
            Zv = np.array(dequantise(np.asarray(ZV[b, g, :Lb, :], np.float64), sv))
            # reduced-rank tokens keep only their leading r_low latent components
            low = imp[b, g, :Lb] < tau
            Zk[low, r_low:] = 0.0
            Zv[low, r_low:] = 0.0
            K = np.zeros((Lb, d))
            V = np.zeros((Lb, d))
            for t in range(Lb):
                m = 0 if (n_visual == 0 or t < n_visual) else 1
                fk = BK[m][g] if n_visual else BK[g]
                fv = BV[m][g] if n_visual else BV[g]
                K[t] = Zk[t] @ np.asarray(fk, np.float64)
                V[t] = Zv[t] @ np.asarray(fv, np.float64)
            for h in range(g * G, (g + 1) * G):
                s = (K @ q[b, h]) / math.sqrt(d)
                mx = s.max()
                e = np.exp(s - mx)
                l = e.sum()
                out[b, h] = (e / l) @ V
                lse[b, h] = mx + math.log(l)
                mass[b, g, :Lb] += e / l
    new_imp = imp.copy()
    for b in range(B):
        Lb = int(seqlens[b])
        new_imp[b, :, :Lb] = beta * imp[b, :, :Lb] + (1.0 - beta) * mass[b, :, :Lb]
    return out, lse, mass, new_imp


def decode_attention_shared(q, ZK, ZV, DK, DV, seqlens, n_kv_heads: int, ZK_scale=None,
                            ZV_scale=None):
    """Cross-head shared latent ("AttentionPack", Metodologia 2.A, multi-head
    compression: the key (value) rows of all heads are concatenated along the head axis
    and factored once, so a token keeps one latent of rank R for every head and one
    decompression matrix of R x (H d) serves them all).

    q [B][Hq][d]; ZK, ZV [B][L_cap][R] (decoded codes); scales [B][L_cap] or None;
    DK, DV [R][n_kv_heads * d]; seqlens [B]. KV head g's keys are Z_K D_K[:, g d:(g+1) d]
    (its values likewise); query head h reads KV head h // G. Returns out [B][Hq][d] and
    lse [B][Hq]. Reading: the concatenation order is head-major (head g owns columns
    g d .. g d + d - 1 of D)."""
    q = np.asarray(q, np.float64)
    B, Hq, d = q.shape
    G = Hq // n_kv_heads
    out = np.zeros((B, Hq, d))
    lse = np.full((B, Hq), -np.inf)
    for b in range(B):
        Lb = int(seqlens[b])
        if Lb == 0:
            continue
        sk = None if ZK_scale is None else ZK_scale[b, :Lb]
        sv = None if ZV_scale is None else ZV_scale[b, :Lb]
        Zk = dequantise(np.asarray(ZK[b, :Lb, :], np.float64), sk)
        Zv = dequantise(np.asarray(ZV[b, :Lb, :], np.float64), sv)
        Kall = Zk @ np.asarray(DK, np.float64)        # Lb x (H d): every head at once
        Vall = Zv @ np.asarray(DV, np.float64)
        for h in range(Hq):
            g = h // G
            K = Kall[:, g * d:(g + 1) * d]
            V = Vall[:, g * d:(g + 1) * d]
            s = (K @ q[b, h]) / math.sqrt(d)
            m = s.max()
            e = np.exp(s - m)
            l = e.sum()
            out[b, h] = (e / l) @ V
            lse[b, h] = m + math.log(l)
    return out, lse


def decode_attention_reassociated(q, ZK, ZV, BK, BV, seqlens, ZK_scale=None, ZV_scale=None):
    """The same attention computed without rebuilding K, V: scores as
    (q B_K^T) Z_K^T and output as (p Z_V) B_V. Exactly equal in real arithmetic;
    an independent second form used to pin the reconstruction."""
    q = np.asarray(q, np.float64)
    B, Hq, d = q.shape
    Hkv = ZK.shape[1]
    G = Hq // Hkv
    out = np.zeros((B, Hq, d))
    lse = np.full((B, Hq), -np.inf)
    for b in range(B):
        Lb = int(seqlens[b])
        if Lb == 0:
            continue
        for h in range(Hq):
            g = h // G
            sk = None if ZK_scale is None else ZK_scale[b, g, :Lb]
            sv = None if ZV_scale is None else ZV_scale[b, g, :Lb]
            Zk = dequantise(np.asarray(ZK[b, g, :Lb, :], np.float64), sk)
            Zv = dequantise(np.asarray(ZV[b, g, :Lb, :], np.float64), sv)
            qt = np.asarray(BK[g], np.float64) @ q[b, h]     # r
            s = (Zk @ qt) / math.sqrt(d)
            m = s.max()
            e = np.exp(s - m)
            l = e.sum()
            zbar = (e / l) @ Zv                                # r
            out[b, h] = zbar @ np.asarray(BV[g], np.float64)
            lse[b, h] = m + math.log(l)
    return out, lse


def split_partials(q, ZK, ZV, BK, BV, seqlens, chunk: int, n_splits: int,
                   ZK_scale=None, ZV_scale=None):
    """Flash-Decoding partials: split s covers tokens [s*chunk, min((s+1)*chunk, L_b)).
    Returns o [B][Hq][S][d] (each normalised by its own sum) and lse [B][Hq][S];
    an empty split has o = 0 and lse = -inf."""
    q = np.asarray(q, np.float64)
    B, Hq, d = q.shape
    Hkv = ZK.shape[1]
    G = Hq // Hkv
    o = np.zeros((B, Hq, n_splits, d))
    lse = np.full((B, Hq, n_splits), -np.inf)
    for b in range(B):
        Lb = int(seqlens[b])
        for h in range(Hq):
            g = h // G
            for s_idx in range(n_splits):
                t0, t1 = s_idx * chunk, min((s_idx + 1) * chunk, Lb)
                if t1 <= t0:
                    continue
                sk = None if ZK_scale is None else ZK_scale[b, g, t0:t1]
                sv = None if ZV_scale is None else ZV_scale[b, g, t0:t1]
                K = dequantise(np.asarray(ZK[b, g, t0:t1], np.float64), sk) @ BK[g]
                V = dequantise(np.asarray(ZV[b, g, t0:t1], np.float64), sv) @ BV[g]
                s = (K @ q[b, h]) / math.sqrt(d)
                m = s.max()
                e = np.exp(s - m)
                l = e.sum()
                o[b, h, s_idx] = (e / l) @ V
                lse[b, h, s_idx] = m + math.log(l)
    return o, lse


def merge_partials(o, lse):
    """LSE merge across splits: LSE = log sum_s exp(lse_s); out = sum_s
    exp(lse_s - LSE) o_s. Splits with lse = -inf contribute nothing; a row whose
    splits are all empty gives out = 0, LSE = -inf."""
    B, Hq, S, d = o.shape
    out = np.zeros((B, Hq, d))
    LSE = np.full((B, Hq), -np.inf)
    for b in range(B):
        for h in range(Hq):
            ls = lse[b, h]
            valid = np.isfinite(ls)
            if not valid.any():
                continue
            m = ls[valid].max()
            tot = np.exp(ls[valid] - m).sum()
            L = m + math.log(tot)
            w = np.exp(ls[valid] - L)
            out[b, h] = (w[:, None] * o[b, h, valid]).sum(axis=0)
            LSE[b, h] = L
    return out, LSE


# --------------------------------------------------------------------------------------
# Append (one new latent row per decode step), with the per-token quantiser
# --------------------------------------------------------------------------------------


def quantise_int8_row(z32: np.ndarray):
    """Symmetric absmax int8: scale = absmax / 127 (fp32, IEEE division), code =
    round-half-even(z / scale) in fp32, clamped to [-127, 127]. All-zero row: scale 1."""
    z32 = np.asarray(z32, dtype=np.float32)
    amax = np.float32(np.max(np.abs(z32))) if z32.size else np.float32(0)
    if amax == 0:
        return np.zeros(z32.shape, np.int8), np.float32(1.0)
    scale = np.float32(amax / np.float32(127.0))
    v = (z32 / scale).astype(np.float32)
    codes = np.clip(np.rint(v), -127, 127).astype(np.int8)
    return codes, scale


def quantise_e4m3_row(z32: np.ndarray):
    """Absmax e4m3: scale = absmax / 448 (fp32), code = RNE-satfinite(z / scale)."""
    z32 = np.asarray(z32, dtype=np.float32)
    amax = np.float32(np.max(np.abs(z32))) if z32.size else np.float32(0)
    if amax == 0:
        return np.zeros(z32.shape, np.uint8), np.float32(1.0)
    scale = np.float32(amax / np.float32(448.0))
    v = (z32 / scale).astype(np.float32)
    return f32_to_e4m3_rne_sat(v), scale


STATUS_APPEND_FULL = 4


def append(ZK, ZV, ZK_scale, ZV_scale, seqlens, zk_new32, zv_new32, latent_dtype: str):
    """Write one new latent row per (batch, KV head) at slot seqlens[b], then
    seqlens[b] += 1. Arrays are stored-format numpy copies (bf16 as uint16 bits,
    e4m3 as uint8 codes); zk_new32/zv_new32 are the new rows as float32 [B][Hkv][r].
    A row whose slot is past the capacity is left untouched and flagged.
    Returns (ZK, ZV, ZK_scale, ZV_scale, seqlens, status)."""
    ZK, ZV = ZK.copy(), ZV.copy()
    ZK_scale = None if ZK_scale is None else ZK_scale.copy()
    ZV_scale = None if ZV_scale is None else ZV_scale.copy()
    seqlens = np.asarray(seqlens, np.int32).copy()
    B, Hkv, L_cap, r = ZK.shape
    status = 0
    for b in range(B):
        slot = int(seqlens[b])
        if slot < 0 or slot >= L_cap:
            status |= STATUS_APPEND_FULL
            continue
        for g in range(Hkv):
            for Z, S, znew in ((ZK, ZK_scale, zk_new32), (ZV, ZV_scale, zv_new32)):
                row = np.asarray(znew[b, g], np.float32)
                if latent_dtype == "f32":
                    Z[b, g, slot] = row
                elif latent_dtype == "bf16":
                    Z[b, g, slot] = f32_to_bf16_bits_rne(row)
                elif latent_dtype == "i8":
                    c, s = quantise_int8_row(row)
                    Z[b, g, slot] = c
                    S[b, g, slot] = s
                elif latent_dtype == "e4m3":
                    c, s = quantise_e4m3_row(row)
                    Z[b, g, slot] = c
                    S[b, g, slot] = s
                else:
                    raise ValueError(latent_dtype)
        seqlens[b] = slot + 1
    return ZK, ZV, ZK_scale, ZV_scale, seqlens, status


def project(x, AK, AV):
    """The new token's latents for every (batch row, KV head): z_K = x A_K,g and
    z_V = x A_V,g (the cached latent is the token's hidden state times the head's down
    factor, W = A B: "WSVD: Weighted Low-Rank Approximation for Fast and Efficient
    Execution of Low-Precision Vision-Language Models", section 2.A), in fp64.
    x [B][d_model], A [Hkv][d_model][r] -> two arrays [B][Hkv][r]."""
    x = np.asarray(x, np.float64)
    AK = np.asarray(AK, np.float64)
    AV = np.asarray(AV, np.float64)
    return np.einsum("bi,gir->bgr", x, AK), np.einsum("bi,gir->bgr", x, AV)


def project_append(ZK, ZV, ZK_scale, ZV_scale, seqlens, x, AK, AV, latent_dtype: str):
    """Fused projection + append: project, take the fp32 value of each latent (the
    precision the kernel stores and quantises in), then append as above."""
    zk, zv = project(x, AK, AV)
    return append(ZK, ZV, ZK_scale, ZV_scale, seqlens, zk.astype(np.float32),
                  zv.astype(np.float32), latent_dtype)
