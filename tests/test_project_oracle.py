"""Pins of the oracle's latent projection (the fused projection + append step):
identity factors give the hidden state back, a pure-Python loop agrees on tiny shapes,
the projection is linear, and projection + append with identity factors is exactly
append of the hidden state. A transposed-factor mistake is caught by the loop pin."""
import numpy as np

from oracle import lrkv_oracle as orc


def _loop_project(x, A):
    B, D = x.shape
    H, _, r = A.shape
    z = [[[0.0] * r for _ in range(H)] for _ in range(B)]
    for b in range(B):
        for g in range(H):
            for k in range(r):
                z[b][g][k] = sum(float(x[b][i]) * float(A[g][i][k]) for i in range(D))
    return np.array(z)


def test_identity_factors_return_the_hidden_state():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((3, 8))
    A = np.stack([np.eye(8), 2 * np.eye(8)])
    zk, zv = orc.project(x, A, A[::-1])
    np.testing.assert_array_equal(zk[:, 0], x)
    np.testing.assert_array_equal(zk[:, 1], 2 * x)
    np.testing.assert_array_equal(zv[:, 0], 2 * x)


def test_pure_python_loop_agrees():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((2, 5))
    AK = rng.standard_normal((3, 5, 4))
    AV = rng.standard_normal((3, 5, 4))
    zk, zv = orc.project(x, AK, AV)
    np.testing.assert_allclose(zk, _loop_project(x, AK), rtol=0, atol=1e-12)
    np.testing.assert_allclose(zv, _loop_project(x, AV), rtol=0, atol=1e-12)
    # the mistake of contracting over the wrong factor axis is caught
    bad = np.einsum("bi,gri->bgr", x[:, :4], AK[:, :4, :4])
    assert not np.allclose(bad, _loop_project(x[:, :4], AK[:, :4, :4]))


def test_projection_is_linear():
    rng = np.random.default_rng(5)
    x1, x2 = rng.standard_normal((2, 4, 16))
    A = rng.standard_normal((2, 16, 8))
    a1, _ = orc.project(x1, A, A)
    a2, _ = orc.project(x2, A, A)
    a12, _ = orc.project(3 * x1 - x2, A, A)
    np.testing.assert_allclose(a12, 3 * a1 - a2, rtol=0, atol=1e-12)


def test_project_append_with_identity_factors_is_append():
    rng = np.random.default_rng(6)
    B, H, L, r = 2, 2, 6, 8
    x = (rng.standard_normal((B, r)) * 3).astype(np.float32).astype(np.float64)
    A = np.stack([np.eye(r)] * H)
    for lat in ("f32", "bf16", "i8", "e4m3"):
        zdt = {"f32": np.float32, "bf16": np.uint16, "i8": np.int8, "e4m3": np.uint8}[lat]
        ZK = np.zeros((B, H, L, r), zdt)
        ZV = np.zeros((B, H, L, r), zdt)
        SK = np.ones((B, H, L), np.float32) if lat in ("i8", "e4m3") else None
        SV = None if SK is None else SK.copy()
        seq = np.array([1, 5], np.int32)
        got = orc.project_append(ZK, ZV, SK, SV, seq, x, A, A, lat)
        rows = np.stack([x.astype(np.float32)] * H, axis=1)
        want = orc.append(ZK, ZV, SK, SV, seq, rows, rows, lat)
        for gv, wv in zip(got, want):
            if gv is None:
                assert wv is None
            else:
                np.testing.assert_array_equal(np.asarray(gv), np.asarray(wv))
