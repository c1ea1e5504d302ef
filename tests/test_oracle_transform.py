"""Pins of the oracle's key pre-transform and calibration."""
import numpy as np
import scipy.linalg

import oracle

C128 = np.float32(1.0 / np.sqrt(128.0))


def test_hadamard_rows_match_scipy_sylvester():
    eye = np.eye(128, dtype=np.float32)[:, None, :]     # 128 tokens, 1 head
    y = oracle.transform_keys(eye, np.ones((1, 128), np.float32), hadamard=True)[:, 0, :]
    H = scipy.linalg.hadamard(128).astype(np.float64)
    np.testing.assert_array_equal(y.astype(np.float64), H.T * np.float64(C128))


def test_hadamard_is_orthogonal():
    eye = np.eye(128, dtype=np.float32)[:, None, :]
    y = oracle.transform_keys(eye, np.ones((1, 128), np.float32), hadamard=True)[:, 0, :]
    Hm = np.rint(y.astype(np.float64) / np.float64(C128))
    np.testing.assert_array_equal(Hm @ Hm.T, 128.0 * np.eye(128))


def test_transform_preserves_dot_products():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((64, 2, 128)).astype(np.float32)
    y = oracle.transform_keys(x, np.ones((2, 128), np.float32), hadamard=True)
    a = np.einsum("thc,thc->th", x.astype(np.float64), x.astype(np.float64))
    b = np.einsum("thc,thc->th", y.astype(np.float64), y.astype(np.float64))
    np.testing.assert_allclose(b, a, rtol=1e-5)


def test_smoothing_multiplies_by_inverse():
    rng = np.random.default_rng(1)
    k = rng.standard_normal((10, 3, 128)).astype(np.float32)
    inv = rng.uniform(0.1, 2.0, (3, 128)).astype(np.float32)
    y = oracle.transform_keys(k, inv, hadamard=False)
    # one fp32 rounding of the exact product
    np.testing.assert_array_equal(y, (k.astype(np.float64) * inv).astype(np.float32))


def _windows():
    L, W, T, H, D = 2, 3, 6, 2, 128
    k = np.zeros((L, W, T, H, D), np.float32)
    v = np.zeros((L, W, T, H, D), np.float32)
    rng = np.random.default_rng(2)
    A = rng.uniform(0.5, 9.0, (L, H, D)).astype(np.float32)
    for l in range(L):
        for h in range(H):
            for c in range(D):
                w, t = rng.integers(0, W), rng.integers(1, T)
                k[l, w, t, h, c] = A[l, h, c] * (1 if rng.random() < 0.5 else -1)
    k[:, :, 0] = 50.0            # the sink at position 0 of each window
    A[:, :, 7] = 0.0
    k[:, :, 1:, :, 7] = 0.0      # channel 7: zero outside the sink
    v[1, 2, 3, 1, 5] = -13.0
    v[0, 0, 0, 0, 0] = 4.0
    return k, v, A


def test_calibrate_excludes_position_zero():
    k, v, A = _windows()
    s, inv, gk, gv = oracle.calibrate(k, v, exclude_pos0=True, hadamard=False)
    want_s = np.where(A > 0, np.sqrt(A.astype(np.float64)).astype(np.float32), np.float32(1))
    np.testing.assert_array_equal(s, want_s)
    np.testing.assert_array_equal(inv, (1.0 / want_s.astype(np.float64)).astype(np.float32))
    # per-tensor key scale: amax of the transformed tensor, sink included
    amax = (np.float32(50.0) * inv).max(axis=(1, 2))
    np.testing.assert_array_equal(gk, (amax.astype(np.float64) / 2688.0).astype(np.float32))
    np.testing.assert_array_equal(gv, np.array([4.0 / 2688.0, 13.0 / 2688.0], np.float32))


def test_calibrate_including_position_zero():
    k, v, A = _windows()
    s, inv, gk, gv = oracle.calibrate(k, v, exclude_pos0=False, hadamard=False)
    np.testing.assert_array_equal(s, np.full_like(s, np.sqrt(np.float32(50.0))))


def test_calibrate_all_zero_gives_unit_scales():
    z = np.zeros((1, 1, 4, 1, 128), np.float32)
    s, inv, gk, gv = oracle.calibrate(z, z)
    assert np.all(s == 1) and np.all(inv == 1) and gk[0] == 1 and gv[0] == 1


def test_calibrate_native_basis_keeps_keys_unsmoothed():
    # "NVFP4 attention cache on W4A4 Qwen3-8B", results table row "NVFP4 K
    # only, native basis": no smoothing, so
    # s = inv = 1 and the key tensor scale is the plain absmax over every
    # calibration token (the sink of _windows at 50 included)
    k, v, A = _windows()
    s, inv, gk, gv = oracle.calibrate(k, v, hadamard=False, smooth=False)
    assert np.all(s == 1) and np.all(inv == 1)
    np.testing.assert_array_equal(gk, np.full(2, np.float32(50.0 / 2688.0)))
    np.testing.assert_array_equal(gv, np.array([4.0 / 2688.0, 13.0 / 2688.0], np.float32))


def test_calibrate_native_basis_with_rotation_against_scipy():
    # with the rotation and no smoothing the key scale is max |H k| / sqrt(128)
    # over all tokens / 2688; H from scipy (fp64), so compare to a few ulps
    from scipy.linalg import hadamard
    rng = np.random.default_rng(7)
    k = rng.standard_normal((1, 2, 8, 2, 128)).astype(np.float32)
    v = rng.standard_normal((1, 2, 8, 2, 128)).astype(np.float32)
    s, inv, gk, gv = oracle.calibrate(k, v, hadamard=True, smooth=False)
    assert np.all(s == 1)
    rot = k.astype(np.float64) @ hadamard(128).T / np.sqrt(128.0)
    np.testing.assert_allclose(gk[0], np.abs(rot).max() / 2688.0, rtol=4e-7)
    assert gv[0] == np.float32(np.abs(v).max() / 2688.0)
