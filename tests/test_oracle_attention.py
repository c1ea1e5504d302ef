"""Pins of the oracle's attention against a separately written formula."""
import numpy as np
import pytest
import scipy.linalg
import scipy.special

import oracle


def naive(q, k, v, G):
    """softmax(q k^T / sqrt(D)) v per query head, kv head = q head // G (fp64)."""
    Tq, Hq, D = q.shape
    out = np.empty((Tq, Hq, D))
    for i in range(Tq):
        for hq in range(Hq):
            sc = k[:, hq // G, :] @ q[i, hq] / np.sqrt(D)
            out[i, hq] = scipy.special.softmax(sc) @ v[:, hq // G, :]
    return out


@pytest.mark.parametrize("hadamard", [False, True])
@pytest.mark.parametrize("T", [1, 3, 8])
def test_attention_equals_formula_on_raw_keys(hadamard, T):
    """Smoothing (and rotation) folded into the query gives back q . k."""
    rng = np.random.default_rng(T + 10 * hadamard)
    Hq, Hkv, D = 8, 2, 128
    q = rng.standard_normal((1, Hq, D)).astype(np.float32)
    k = (rng.standard_normal((T, Hkv, D)) * 2).astype(np.float32)
    v = rng.standard_normal((T, Hkv, D))
    s = rng.uniform(0.5, 3.0, (Hkv, D)).astype(np.float32)
    inv = (1.0 / s.astype(np.float64)).astype(np.float32)
    kx = oracle.transform_keys(k, inv, hadamard).astype(np.float64)
    got = oracle.attention(q, T - 1, s, kx, v, hadamard)
    want = naive(q.astype(np.float64), k.astype(np.float64), v, Hq // Hkv)
    np.testing.assert_allclose(got, want, rtol=2e-5, atol=2e-6)


def test_attention_matches_formula_exactly_without_transform():
    rng = np.random.default_rng(5)
    q = rng.standard_normal((3, 8, 128)).astype(np.float32)
    kx = rng.standard_normal((7, 2, 128))
    vx = rng.standard_normal((7, 2, 128))
    s = np.ones((2, 128), np.float32)
    got = oracle.attention(q, 4, s, kx, vx)
    for i in range(3):
        n = min(7, 4 + i + 1)
        want = naive(q[i:i + 1].astype(np.float64), kx[:n], vx[:n], 4)
        np.testing.assert_allclose(got[i:i + 1], want, rtol=1e-12, atol=1e-13)


def test_single_token_returns_its_value():
    rng = np.random.default_rng(6)
    q = rng.standard_normal((1, 8, 128)).astype(np.float32)
    kx = rng.standard_normal((1, 2, 128))
    vx = rng.standard_normal((1, 2, 128))
    out = oracle.attention(q, 0, np.ones((2, 128), np.float32), kx, vx)
    np.testing.assert_array_equal(out[0, :4], np.broadcast_to(vx[0, 0], (4, 128)))
    np.testing.assert_array_equal(out[0, 4:], np.broadcast_to(vx[0, 1], (4, 128)))


def test_equal_keys_give_mean_value():
    rng = np.random.default_rng(7)
    q = rng.standard_normal((1, 4, 128)).astype(np.float32)
    kx = np.broadcast_to(rng.standard_normal((1, 1, 128)), (9, 1, 128)).copy()
    vx = rng.standard_normal((9, 1, 128))
    out = oracle.attention(q, 8, np.ones((1, 128), np.float32), kx, vx)
    np.testing.assert_allclose(out[0], np.broadcast_to(vx.mean(axis=0), (4, 128)), rtol=1e-12, atol=1e-14)


def test_causal_rows_equal_decode_of_prefix():
    rng = np.random.default_rng(8)
    q = rng.standard_normal((4, 8, 128)).astype(np.float32)
    kx = rng.standard_normal((10, 2, 128))
    vx = rng.standard_normal((10, 2, 128))
    s = rng.uniform(0.5, 2, (2, 128)).astype(np.float32)
    full = oracle.attention(q, 6, s, kx, vx, hadamard=True)
    for i in range(4):
        one = oracle.attention(q[i:i + 1], 6 + i, s, kx[: 7 + i], vx[: 7 + i], hadamard=True)
        np.testing.assert_allclose(full[i], one[0], rtol=1e-13, atol=1e-14)
