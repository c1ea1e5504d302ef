"""Pins of the oracle's NVFP4 block quantiser."""
import numpy as np
import pytest

import oracle
from conftest import read_golden

GRID = np.array([float(v) for _, v in read_golden("e2m1_grid.txt")[:8]])


def nearest_code(t):
    """Nearest E2M1 magnitude index of |t| by direct search (ties: even index)."""
    t = np.abs(np.asarray(t, np.float64))
    d = np.abs(t[..., None] - GRID)
    best = d.min(axis=-1, keepdims=True)
    cand = np.where(d == best, np.arange(8), 99)
    even = np.where(cand % 2 == 0, cand, 99).min(axis=-1)
    return np.where(even < 99, even, cand.min(axis=-1))


def exact_scale_block(rng, k, m, ratios):
    """A block whose max is 6*2^k under g = 2^m: then d = 2^k exactly."""
    a = 6.0 * 2.0 ** k
    y = np.empty(16, np.float64)
    y[0] = a
    y[1:1 + len(ratios)] = a * np.asarray(ratios)
    rest = 15 - len(ratios)
    y[1 + len(ratios):] = rng.uniform(-a, a, rest)
    return y.astype(np.float32), np.float32(2.0 ** m)


@pytest.mark.parametrize("k,m", [(0, 0), (3, -2), (-5, -4), (6, 1), (-2, 5)])
def test_absmax_over_24_closed_form(k, m):
    rows = read_golden("absmax24.txt")
    ratios = [float(r) for r, _ in rows]
    want = [int(c) for _, c in rows]
    rng = np.random.default_rng(abs(k * 31 + m) + 100)
    y, g = exact_scale_block(rng, k, m, ratios + [-r for r in ratios])
    codes, sf = oracle.quantize_rows(np.tile(y, 8)[None, :], g)
    codes = codes[0, :16]
    # block scale: a * enc = 2^(k-m) exactly -> E4M3 value 2^(k-m)
    assert oracle.e4m3_value(sf[0, 0]) == 2.0 ** (k - m)
    n = len(ratios)
    np.testing.assert_array_equal(codes[1:1 + n] & 7, want)
    np.testing.assert_array_equal(codes[1 + n:1 + 2 * n] & 7, want)
    assert np.all(codes[1 + n:1 + 2 * n] & 8)          # negative entries keep the sign
    # every entry follows the nearest-value rule on y / d with d = 2^k
    np.testing.assert_array_equal(codes & 7, nearest_code(y.astype(np.float64) / 2.0 ** k))
    small = np.abs(y) < 6.0 * 2.0 ** k / 24
    assert np.all(codes[small] & 7 == 0)


def test_dequant_error_bound_random_blocks():
    rng = np.random.default_rng(1)
    n = 4000
    scale = np.exp(rng.normal(0, 2, (n, 1)))
    y = (rng.standard_normal((n, 128)) * scale).astype(np.float32)
    y[rng.random((n, 128)) < 0.02] *= 30.0             # outliers inside blocks
    g = np.float32(np.abs(y).max() / 2688.0)
    codes, sf = oracle.quantize_rows(y, g)
    x = oracle.dequantize_rows(codes, sf, g)
    d = oracle.e4m3_value(sf).repeat(16, axis=-1) * float(g)
    # one E2M1 step is at most 2 units of d, so the nearest value is within d;
    # the E4M3 rounding of the scale (relative error <= 2^-4) keeps the block
    # maximum within 6.375 d, inside the same bound.
    normal = oracle.e4m3_value(sf).repeat(16, axis=-1) >= 2.0 ** -6
    err = np.abs(x - y.astype(np.float64))
    assert np.all(err[normal] <= d[normal] * (1 + 1e-6))
    rel = np.linalg.norm(x - y) / np.linalg.norm(y)
    assert rel < 0.12


def test_zero_block_and_signed_zero():
    y = np.zeros((1, 128), np.float32)
    y[0, 16:32] = -0.0
    codes, sf = oracle.quantize_rows(y, np.float32(0.5))
    assert np.all(sf == 0)
    assert np.all(codes[0, :16] == 0) and np.all(codes[0, 16:32] == 8)


def test_scale_saturation():
    # block max far beyond the calibrated range: scale saturates at 448 and
    # the entries saturate at +-6
    y = np.zeros((1, 128), np.float32)
    y[0, :16] = np.linspace(-1e4, 1e4, 16)
    codes, sf = oracle.quantize_rows(y, np.float32(1.0))
    assert sf[0, 0] == 0x7E
    assert codes[0, 0] == 15 and codes[0, 15] == 7


def test_blocks_are_independent():
    rng = np.random.default_rng(3)
    y = rng.standard_normal((5, 128)).astype(np.float32) * 3
    g = np.float32(0.01)
    codes, sf = oracle.quantize_rows(y, g)
    perm = rng.permutation(8)
    yp = y.reshape(5, 8, 16)[:, perm].reshape(5, 128)
    cp, sp = oracle.quantize_rows(yp, g)
    np.testing.assert_array_equal(cp.reshape(5, 8, 16), codes.reshape(5, 8, 16)[:, perm])
    np.testing.assert_array_equal(sp, sf[:, perm])


def test_dequantize_is_product_of_format_values():
    rng = np.random.default_rng(4)
    codes = rng.integers(0, 16, (3, 128)).astype(np.uint8)
    sf = rng.integers(0, 0x7F, (3, 8)).astype(np.uint8)
    g = np.float32(0.037)
    x = oracle.dequantize_rows(codes, sf, g)
    grid = np.array([float(v) for _, v in read_golden("e2m1_grid.txt")])
    want = grid[codes] * oracle.e4m3_value(sf).repeat(16, axis=-1) * float(g)
    np.testing.assert_array_equal(x, want)
