"""Pins of the oracle's FP4 query path: the query brought into the keys'
basis (query_rows_fp4), quantised to NVFP4 with an online per-row FP32 scale
(quantize_query), and attended in fp64 (attention_x).

Sources: "NVFP4 attention cache on W4A4 Qwen3-8B" (rstation.ai), setup
paragraph (W4A4: activations in NVFP4) and observation 2 (the smoothing
factor folded into the query); "OSFP4" (paperlayer.ai summary), Problem
bullet, sec. 1 and sec. D.1 (absmax to 6, E4M3 scales per 16, an FP32 scale
above them).
"""
import numpy as np
import scipy.linalg

import oracle


def _rows(n=64, seed=11):
    rng = np.random.default_rng(seed)
    mag = np.exp(rng.uniform(-6, 6, (n, 1)))                 # row magnitudes over many binades
    y = rng.standard_normal((n, 128)) * np.exp(rng.standard_normal(128)) * mag
    return y.astype(np.float32)


def test_quantize_query_is_the_cache_quantiser_row_by_row():
    # with the row's own FP32 scale, every row quantises exactly as the
    # (separately pinned) cache quantiser does
    y = _rows()
    codes, sf, g = oracle.quantize_query(y)
    for r in range(y.shape[0]):
        c1, s1 = oracle.quantize_rows(y[r:r + 1], float(g[r]))
        np.testing.assert_array_equal(codes[r], c1[0])
        np.testing.assert_array_equal(sf[r], s1[0])


def test_row_absmax_maps_to_scale_448_and_code_6():
    # g = amax / (6 * 448): the block holding the row's absmax gets the
    # largest E4M3 scale and the absmax element the largest E2M1 magnitude
    y = _rows(seed=12)
    codes, sf, g = oracle.quantize_query(y)
    for r in range(y.shape[0]):
        i = int(np.argmax(np.abs(y[r])))
        assert sf[r, i // 16] == 0x7E, (r, sf[r, i // 16])
        assert codes[r, i] & 7 == 7 and (codes[r, i] >> 3) == (y[r, i] < 0)
    assert np.all(sf <= 0x7E)                                # nothing above 448
    assert np.all(oracle.e4m3_value(sf) * g[:, None] * 6 <= np.abs(y).max(axis=1)[:, None] * (1 + 2 ** -20))


def test_power_of_two_scaling_moves_only_the_row_scale():
    y = _rows(seed=13)
    codes, sf, g = oracle.quantize_query(y)
    for k in (-20, -3, 5, 30):
        c2, s2, g2 = oracle.quantize_query(y * np.float32(2.0 ** k))
        np.testing.assert_array_equal(c2, codes)
        np.testing.assert_array_equal(s2, sf)
        np.testing.assert_array_equal(g2, g * np.float32(2.0 ** k))


def test_dequantised_query_within_the_nvfp4_error_bound():
    y = _rows(seed=14)
    codes, sf, g = oracle.quantize_query(y)
    x = oracle.dequantize_query(codes, sf, g)
    yb = y.astype(np.float64).reshape(-1, 8, 16)
    d = (oracle.e4m3_value(sf) * g[:, None].astype(np.float64))[..., None]     # block step
    a = np.abs(yb).max(axis=-1, keepdims=True)
    # the largest E2M1 gap is 2 (between 4 and 6): half of it, times the
    # step; a block whose scale rounded down may also saturate at 6 d
    bound = d * (1 + 1e-6) + np.maximum(0.0, a - 6 * d)
    assert np.all(np.abs(x.reshape(yb.shape) - yb) <= bound)
    # and the relative error of the whole query is that of 4-bit codes
    rel = np.linalg.norm(x - y, axis=1) / np.linalg.norm(y, axis=1)
    assert rel.max() < 0.2


def test_zero_row_and_zero_block():
    y = _rows(4, seed=15)
    y[1] = 0.0
    y[2, 16:32] = 0.0
    codes, sf, g = oracle.quantize_query(y)
    assert g[1] == 1.0 and not codes[1].any() and not sf[1].any()
    assert sf[2, 1] == 0 and not (codes[2, 16:32] & 7).any()
    np.testing.assert_array_equal(oracle.dequantize_query(codes, sf, g)[1], 0.0)


def test_query_rows_fp4_transform():
    rng = np.random.default_rng(16)
    Tq, Hq, Hkv = 3, 8, 2
    q = rng.standard_normal((Tq, Hq, 128)).astype(np.float32)
    s = np.exp(rng.standard_normal((Hkv, 128))).astype(np.float32)
    # smoothing only: q * s of the query head's kv head, exactly
    y = oracle.query_rows_fp4(q, s)
    for hq in range(Hq):
        np.testing.assert_array_equal(y[:, hq], q[:, hq] * s[hq // 4])
    # with the rotation: H (q * s) / sqrt(128) (scipy's Sylvester matrix) to fp32 rounding
    yh = oracle.query_rows_fp4(q, s, hadamard=True).astype(np.float64)
    H = scipy.linalg.hadamard(128)
    for hq in range(Hq):
        want = (q[:, hq].astype(np.float64) * s[hq // 4]) @ H.T / np.sqrt(128.0)
        scale = np.abs(q[:, hq] * s[hq // 4]).sum(axis=1, keepdims=True) / np.sqrt(128.0)
        assert np.all(np.abs(yh[:, hq] - want) <= 8 * 2.0 ** -24 * scale)
    # with a KLT basis that permutes channels: the permuted q * s, exactly
    perm = [rng.permutation(128) for _ in range(Hkv)]
    U = np.zeros((Hkv, 128, 128), np.float32)
    for h in range(Hkv):
        U[h, perm[h], np.arange(128)] = 1.0
    yk = oracle.query_rows_fp4(q, s, U=U)
    for hq in range(Hq):
        np.testing.assert_array_equal(yk[:, hq], (q[:, hq] * s[hq // 4])[:, perm[hq // 4]])


def test_attention_x_matches_attention_and_closed_forms():
    rng = np.random.default_rng(17)
    T, Tq, Hq, Hkv = 40, 5, 4, 2
    q = rng.standard_normal((Tq, Hq, 128)).astype(np.float32)
    s = np.exp(0.3 * rng.standard_normal((Hkv, 128))).astype(np.float32)
    kx = rng.standard_normal((T, Hkv, 128))
    vx = rng.standard_normal((T, Hkv, 128))
    # given the fp64 transformed query, the same numbers as the (pinned) attention
    qx = q.astype(np.float64) * np.repeat(s, 2, axis=0).astype(np.float64)[None]
    np.testing.assert_array_equal(oracle.attention_x(qx, 30, kx, vx), oracle.attention(q, 30, s, kx, vx))
    # one visible key: the output is its value
    out = oracle.attention_x(qx[:1], 0, kx, vx)
    for hq in range(Hq):
        np.testing.assert_allclose(out[0, hq], vx[0, hq // 2], rtol=0, atol=1e-15)
    # a zero query weighs the visible keys equally; head hq reads kv head hq // G
    out = oracle.attention_x(np.zeros((Tq, Hq, 128)), 10, kx, vx)
    for i in range(Tq):
        for hq in range(Hq):
            np.testing.assert_allclose(out[i, hq], vx[:11 + i, hq // 2].mean(axis=0), rtol=0, atol=1e-13)
