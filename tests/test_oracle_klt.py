"""Pins of the oracle's static per-head KLT ("NVFP4 attention cache on W4A4
Qwen3-8B", results table rows "K: static per-head KLT" and "K: static KLT +
smoothing"): the transform y' = U^T y as a fixed fp32 fused multiply-add
chain, the basis as the eigenvectors of the keys' second-moment matrix.
"""
import numpy as np

import oracle


def test_klt_apply_permutation_is_exact_and_not_transposed():
    # U[c][i] = 1 where c = perm[i]: output i must be input perm[i], exactly
    rng = np.random.default_rng(3)
    perm = rng.permutation(128)
    U = np.zeros((128, 128), np.float32)
    U[perm, np.arange(128)] = 1.0
    y = rng.standard_normal((5, 128)).astype(np.float32)
    np.testing.assert_array_equal(oracle.klt_apply(y, U), y[:, perm])
    # the identity leaves the rows unchanged
    np.testing.assert_array_equal(oracle.klt_apply(y, np.eye(128, dtype=np.float32)), y)


def test_klt_apply_against_fp64_product():
    rng = np.random.default_rng(4)
    q, _ = np.linalg.qr(rng.standard_normal((128, 128)))
    U = q.astype(np.float32)
    y = (rng.standard_normal((64, 128)) * np.exp(rng.standard_normal(128))).astype(np.float32)
    got = oracle.klt_apply(y, U).astype(np.float64)
    want = y.astype(np.float64) @ U.astype(np.float64)
    # 128 roundings of partial sums bounded by sum |U||y|
    bound = 128 * 2.0 ** -24 * (np.abs(y).astype(np.float64) @ np.abs(U).astype(np.float64))
    assert np.all(np.abs(got - want) <= bound)


def test_klt_basis_recovers_a_known_basis():
    # rows a_i * q_i (columns of a known orthogonal Q) with distinct a_i: the
    # second moment is Q diag(a^2 / N) Q^T, so the basis is Q up to order/sign
    rng = np.random.default_rng(5)
    Q, _ = np.linalg.qr(rng.standard_normal((128, 128)))
    a = np.linspace(10.0, 1.0, 128)
    y = (Q * a).T                                        # [128 rows][128]
    U, w = oracle.klt_basis(y)
    np.testing.assert_allclose(w, a ** 2 / 128.0, rtol=1e-9)
    np.testing.assert_allclose(np.abs(U.T @ Q), np.eye(128), atol=1e-8)
    # sign convention: the largest-magnitude component of every vector is positive
    assert np.all(U[np.argmax(np.abs(U), axis=0), np.arange(128)] > 0)


def test_calibrate_klt_basis_properties_and_scales():
    rng = np.random.default_rng(6)
    L, W, T, H = 1, 2, 40, 2
    sigma = np.exp(rng.standard_normal((H, 128)))
    k = (rng.standard_normal((L, W, T, H, 128)) * sigma).astype(np.float32)
    k[:, :, 0] *= 40.0                                   # a sink at position 0 of each window
    v = rng.standard_normal((L, W, T, H, 128)).astype(np.float32)
    s, inv, U, ev = oracle.calibrate_klt(k, v, exclude_pos0=True)
    for h in range(H):
        u = U[0, h].astype(np.float64)
        np.testing.assert_allclose(u.T @ u, np.eye(128), atol=2e-6)
        assert np.all(np.diff(ev[0, h]) <= 0)
        # U diagonalises the second moment of the smoothed keys without the sink
        y = oracle.transform_keys(k[0, :, 1:].reshape(-1, H, 128), inv[0])[:, h].astype(np.float64)
        C = y.T @ y / y.shape[0]
        D = u.T @ C @ u
        assert np.abs(D - np.diag(np.diag(D))).max() <= 1e-5 * np.abs(np.diag(D)).max()
    # with U = identity the scales are those of plain smoothing
    eye = np.broadcast_to(np.eye(128, dtype=np.float32), U.shape).copy()
    gk, gv = oracle.klt_tensor_scales(k, v, inv, eye)
    _, _, gk0, gv0 = oracle.calibrate(k, v, exclude_pos0=True, hadamard=False)
    np.testing.assert_array_equal(gk, gk0)
    np.testing.assert_array_equal(gv, gv0)
