"""CPU oracle of the NVFP4 attention cache -- TEST INFRASTRUCTURE ONLY.

The arithmetic lives in ``kvq_oracle.c`` (plain C: fp32 quantiser steps in a
fixed order, fp64 attention).  This module compiles it with gcc, loads it with
ctypes and marshals numpy arrays; it computes nothing itself.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` import this package.  The CUDA library (``bit_attention_decode_b200``)
never imports it and it never imports the library.

Parity status of each function (the pins live in ``tests/test_oracle_*.py``):
  e2m1_encode / e2m1_value   pinned (grid golden file, exhaustive brute force)
  e4m3_encode / e4m3_value   pinned (exhaustive brute force, torch float8 cast)
  transform_keys             pinned (scipy Hadamard, H H^T = 128 I, invariance)
  calibrate                  pinned (hand-built windows with known maxima)
  quantize_rows              pinned (absmax/24 closed form, exact-scale blocks,
                             error bound, brute-force per-block search)
  dequantize_rows            pinned (products of the pinned format values)
  attention                  pinned (numpy/scipy softmax formula, one token,
                             equal keys, smoothing invariance)
  klt_apply / klt_basis /    pinned (permutation, fp64 product bound, known
  calibrate_klt              basis, diagonalised second moment)
  quantize_query /           pinned (reduction to quantize_rows row by row,
  query_rows_fp4             row absmax -> scale 448 and code 6, power-of-two
                             invariance, error bound, zero row)
  attention_x                pinned (equals attention on the fp64 transformed
                             query; one visible key; equal scores)
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kvq_oracle.c")
_LIB_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_LIB_DIR, "libkvq_oracle.so")
_lock = threading.Lock()
_lib = None

HEAD_DIM = 128
BLOCK = 16

CFLAGS = ["-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
          "-fPIC", "-shared", "-lm"]


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/_build/libkvq_oracle.so``."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    os.makedirs(_LIB_DIR, exist_ok=True)
    tmp = _LIB + f".tmp{os.getpid()}"
    subprocess.run(["gcc", *CFLAGS, _SRC, "-o", tmp], check=True)
    os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i64, i32, f32 = ctypes.c_int64, ctypes.c_int, ctypes.c_float
        lib.oracle_e2m1_value.restype = ctypes.c_double
        lib.oracle_e2m1_value.argtypes = [ctypes.c_uint32]
        lib.oracle_e4m3_value.restype = ctypes.c_double
        lib.oracle_e4m3_value.argtypes = [ctypes.c_uint32]
        lib.oracle_e2m1_encode_n.argtypes = [P, P, i64]
        lib.oracle_e4m3_encode_n.argtypes = [P, P, i64]
        lib.oracle_transform_keys.argtypes = [P, P, i64, i32, i32, P]
        lib.oracle_calibrate.argtypes = [P, P, i32, i32, i32, i32, i32, i32, i32, P, P, P, P]
        lib.oracle_klt_apply.argtypes = [P, P, ctypes.c_int64, P]
        lib.oracle_quantize_rows.argtypes = [P, i64, f32, P, P]
        lib.oracle_dequantize_rows.argtypes = [P, P, i64, f32, P]
        lib.oracle_attention.argtypes = [P, i32, i32, i32, i32, P, i32, P, P, i32, P]
        lib.oracle_quantize_query_rows.argtypes = [P, i64, P, P, P]
        lib.oracle_attention_x.argtypes = [P, i32, i32, i32, i32, P, P, i32, P]
        for name in ("oracle_e2m1_encode_n", "oracle_e4m3_encode_n", "oracle_transform_keys",
                     "oracle_calibrate", "oracle_klt_apply", "oracle_quantize_rows", "oracle_dequantize_rows",
                     "oracle_attention", "oracle_quantize_query_rows", "oracle_attention_x"):
            getattr(lib, name).restype = None
        _lib = lib
        return lib


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data_as(ctypes.c_void_p)


def _f32(x):
    """Host fp32 copy of an array or tensor (bf16 widens exactly)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.float32).contiguous().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(x, dtype=np.float32)


# ---------------------------------------------------------------- formats
def e2m1_value(codes) -> np.ndarray:
    lib = _load()
    codes = np.asarray(codes, dtype=np.uint32)
    table = np.array([lib.oracle_e2m1_value(c) for c in range(16)])
    return table[codes & 15]


def e4m3_value(codes) -> np.ndarray:
    lib = _load()
    codes = np.asarray(codes, dtype=np.uint32)
    table = np.array([lib.oracle_e4m3_value(c) for c in range(256)])
    return table[codes & 255]


def e2m1_encode(x) -> np.ndarray:
    x, px = _c(_f32(x), np.float32)
    out = np.empty(x.shape, np.uint8)
    _load().oracle_e2m1_encode_n(px, out.ctypes.data_as(ctypes.c_void_p), x.size)
    return out


def e4m3_encode(x) -> np.ndarray:
    x, px = _c(_f32(x), np.float32)
    out = np.empty(x.shape, np.uint8)
    _load().oracle_e4m3_encode_n(px, out.ctypes.data_as(ctypes.c_void_p), x.size)
    return out


# ---------------------------------------------------------------- method steps
def calibrate(k_calib, v_calib, exclude_pos0: bool = True, hadamard: bool = False, smooth: bool = True):
    """k/v_calib [L][W][T][H][D] -> (s, inv_s [L][H][D] fp32, g_K, g_V [L] fp32).
    smooth=False keeps the keys in their native basis (s = 1)."""
    k, pk = _c(_f32(k_calib), np.float32)
    v, pv = _c(_f32(v_calib), np.float32)
    L, W, T, H, D = k.shape
    assert D == HEAD_DIM and v.shape == k.shape
    s = np.empty((L, H, D), np.float32)
    inv = np.empty((L, H, D), np.float32)
    gk = np.empty(L, np.float32)
    gv = np.empty(L, np.float32)
    P = ctypes.c_void_p
    _load().oracle_calibrate(pk, pv, L, W, T, H, int(bool(exclude_pos0)), int(bool(hadamard)), int(bool(smooth)),
                             s.ctypes.data_as(P), inv.ctypes.data_as(P),
                             gk.ctypes.data_as(P), gv.ctypes.data_as(P))
    return s, inv, gk, gv


def transform_keys(k, inv_s, hadamard: bool = False) -> np.ndarray:
    """k [n][H][D], inv_s [H][D] -> transformed keys [n][H][D] (fp32)."""
    k, pk = _c(_f32(k), np.float32)
    inv, pi = _c(_f32(inv_s), np.float32)
    n, H, D = k.shape
    y = np.empty_like(k)
    _load().oracle_transform_keys(pk, pi, n, H, int(bool(hadamard)), y.ctypes.data_as(ctypes.c_void_p))
    return y


def quantize_rows(y, g: float):
    """y [..., D] fp32 -> (codes [..., D] uint8 one code per byte, sf [..., D/16] uint8)."""
    y, py = _c(_f32(y), np.float32)
    n = y.size // HEAD_DIM
    codes = np.empty(y.shape, np.uint8)
    sf = np.empty(y.shape[:-1] + (HEAD_DIM // BLOCK,), np.uint8)
    P = ctypes.c_void_p
    _load().oracle_quantize_rows(py, n, float(g), codes.ctypes.data_as(P), sf.ctypes.data_as(P))
    return codes, sf


def dequantize_rows(codes, sf, g: float) -> np.ndarray:
    codes, pc = _c(codes, np.uint8)
    sf, ps = _c(sf, np.uint8)
    x = np.empty(codes.shape, np.float64)
    _load().oracle_dequantize_rows(pc, ps, codes.size // HEAD_DIM, float(g),
                                   x.ctypes.data_as(ctypes.c_void_p))
    return x


def attention(q, q_start: int, s, kx, vx, hadamard: bool = False) -> np.ndarray:
    """q [Tq][Hq][D]; s [Hkv][D]; kx, vx [T][Hkv][D] fp64 -> out [Tq][Hq][D] fp64."""
    q, pq = _c(_f32(q), np.float32)
    s, ps = _c(_f32(s), np.float32)
    kx, pk = _c(kx, np.float64)
    vx, pv = _c(vx, np.float64)
    Tq, Hq, D = q.shape
    T, Hkv, _ = kx.shape
    out = np.empty((Tq, Hq, D), np.float64)
    _load().oracle_attention(pq, Tq, int(q_start), Hq, Hkv, ps, int(bool(hadamard)), pk, pv, T,
                             out.ctypes.data_as(ctypes.c_void_p))
    return out


def round_bf16(x) -> np.ndarray:
    """fp32 -> nearest bf16 value (ties to even), returned as fp32.  A bf16 is
    the upper half of an fp32 encoding; rounding adds half a unit of the kept
    part (0x7FFF, plus one when the kept part is odd) before the lower half is
    dropped.  The keys of the mixed cache ([P1] results table, row "NVFP4 V
    only": keys in BF16) are stored this way."""
    b = np.ascontiguousarray(x, np.float32).view(np.uint32).astype(np.uint64)
    r = (b + 0x7FFF + ((b >> 16) & 1)) & 0xFFFF0000
    return r.astype(np.uint32).view(np.float32)


def klt_apply(y, U) -> np.ndarray:
    """y [..., 128] fp32, U [128][128] fp32 -> U^T y per row, each output one
    fp32 fused multiply-add chain over c = 0..127 (the library's order)."""
    y, py = _c(_f32(y), np.float32)
    U, pu = _c(_f32(U), np.float32)
    n = y.size // HEAD_DIM
    out = np.empty_like(y)
    _load().oracle_klt_apply(py, pu, n, out.ctypes.data_as(ctypes.c_void_p))
    return out


def klt_basis(y) -> np.ndarray:
    """Static per-head KLT basis ("NVFP4 attention cache on W4A4 Qwen3-8B",
    results table rows "K: static per-head KLT" and "K: static KLT +
    smoothing"): the eigenvectors of the second-moment matrix
    C = sum_t y_t y_t^T / N of the (smoothed) calibration keys y [N][128], in
    fp64, ordered by decreasing eigenvalue, each signed so that its component
    of largest magnitude is positive.  Returns (U [128][128] fp64 with
    U[c][i] = component c of vector i, eigenvalues [128] fp64)."""
    y = np.asarray(y, np.float64)
    C = y.T @ y / y.shape[0]
    w, U = np.linalg.eigh(C)
    order = np.argsort(-w, kind="stable")
    w, U = w[order], U[:, order]
    big = np.argmax(np.abs(U), axis=0)
    U = U * np.where(U[big, np.arange(U.shape[1])] < 0, -1.0, 1.0)
    return U, w


def calibrate_klt(k_calib, v_calib, exclude_pos0: bool = True):
    """Smoothing (as calibrate) followed by a KLT basis per (layer, kv head)
    from the smoothed calibration keys, position 0 of each window left out
    when exclude_pos0 (as for the smoothing absmax).
    Returns (s, inv_s, U [L][H][128][128] fp32, eigenvalues [L][H][128])."""
    k = _f32(k_calib)
    s, inv, _, _ = calibrate(k_calib, v_calib, exclude_pos0=exclude_pos0, hadamard=False)
    L, W, T, H, D = k.shape
    t0 = 1 if exclude_pos0 else 0
    U = np.empty((L, H, D, D), np.float32)
    ev = np.empty((L, H, D))
    for l in range(L):
        y = transform_keys(k[l, :, t0:].reshape(-1, H, D), inv[l], False)
        for h in range(H):
            u, w = klt_basis(y[:, h])
            U[l, h], ev[l, h] = u.astype(np.float32), w
    return s, inv, U, ev


def klt_tensor_scales(k_calib, v_calib, inv_s, U):
    """g_K, g_V [L] for keys transformed by smoothing then U (any U, e.g. the
    library's): max |U^T (k * inv_s)| over every calibration token, position 0
    included, / 2688 (1 if zero); g_V as calibrate."""
    k = _f32(k_calib)
    v = _f32(v_calib)
    L, W, T, H, D = k.shape
    gk = np.empty(L, np.float32)
    gv = np.empty(L, np.float32)
    for l in range(L):
        y = transform_keys(k[l].reshape(-1, H, D), inv_s[l], False)
        a = np.float32(0.0)
        for h in range(H):
            a = max(a, np.abs(klt_apply(y[:, h], U[l, h])).max())
        b = np.abs(v[l]).max()
        gk[l] = np.float32(a) / np.float32(2688.0) if a > 0 else np.float32(1.0)
        gv[l] = np.float32(b) / np.float32(2688.0) if b > 0 else np.float32(1.0)
    return gk, gv


# ---------------------------------------------------------------- FP4 queries
def query_rows_fp4(q, s, hadamard: bool = False, U=None) -> np.ndarray:
    """The query in the keys' basis, in fp32, as the FP4 Q.K product
    quantises it: q [Tq][Hq][D], s [Hkv][D] -> [Tq][Hq][D] fp32.
    Query head hq uses kv head hq // G.  Either the key transform with the
    smoothing factor in place of its reciprocal (q * s, then the normalised
    Hadamard-128 when hadamard; [P1] observation 2, [P5]), or, with a KLT
    basis U [Hkv][D][D], q * s followed by U^T as one fp32 fused
    multiply-add chain per output (klt_apply)."""
    q = _f32(q)
    Tq, Hq, D = q.shape
    s = _f32(s)
    G = Hq // s.shape[0]
    rep = np.repeat(s, G, axis=0)
    if U is None:
        return transform_keys(q, rep, hadamard)
    y = transform_keys(q, rep, False)
    out = np.empty_like(y)
    for hq in range(Hq):
        out[:, hq] = klt_apply(y[:, hq], _f32(U)[hq // G])
    return out


def quantize_query(y):
    """Transformed query rows y [..., D] fp32 -> (codes [..., D] one code per
    byte, sf [..., D/16], g [...] fp32): NVFP4 with an FP32 scale per row,
    g = amax(row) / 2688 (1 for a zero row), then the cache's block
    quantiser (oracle_quantize_query_rows)."""
    y, py = _c(_f32(y), np.float32)
    n = y.size // HEAD_DIM
    codes = np.empty(y.shape, np.uint8)
    sf = np.empty(y.shape[:-1] + (HEAD_DIM // BLOCK,), np.uint8)
    g = np.empty(y.shape[:-1], np.float32)
    P = ctypes.c_void_p
    _load().oracle_quantize_query_rows(py, n, codes.ctypes.data_as(P), sf.ctypes.data_as(P), g.ctypes.data_as(P))
    return codes, sf, g


def dequantize_query(codes, sf, g) -> np.ndarray:
    """Exact fp64 value of quantised query rows: val(code) * val(sf) * g."""
    codes = np.asarray(codes)
    step = e4m3_value(np.repeat(np.asarray(sf), BLOCK, axis=-1)) * np.asarray(g, np.float64)[..., None]
    return e2m1_value(codes) * step


def attention_x(qx, q_start: int, kx, vx) -> np.ndarray:
    """Causal GQA attention (as attention) of queries already in the keys'
    basis: qx [Tq][Hq][D] fp64, kx, vx [T][Hkv][D] fp64 -> [Tq][Hq][D] fp64."""
    qx, pq = _c(qx, np.float64)
    kx, pk = _c(kx, np.float64)
    vx, pv = _c(vx, np.float64)
    Tq, Hq, D = qx.shape
    T, Hkv, _ = kx.shape
    out = np.empty((Tq, Hq, D), np.float64)
    _load().oracle_attention_x(pq, Tq, int(q_start), Hq, Hkv, pk, pv, T, out.ctypes.data_as(ctypes.c_void_p))
    return out


# ---------------------------------------------------------------- composites
def quantize_kv(k, v, inv_s, g_k: float, g_v: float, hadamard: bool = False):
    """Quantise one layer's tokens: k, v [n][H][D] -> dict of codes and scales."""
    y = transform_keys(k, inv_s, hadamard)
    kc, ksf = quantize_rows(y, g_k)
    vc, vsf = quantize_rows(_f32(v), g_v)
    return {"kc": kc, "ksf": ksf, "vc": vc, "vsf": vsf}


def decode_reference(q, k, v, s, inv_s, g_k, g_v, hadamard=False, q_start=None):
    """Quantise a sequence's K/V, dequantise, and attend with q [Tq][Hq][D]."""
    qz = quantize_kv(k, v, inv_s, g_k, g_v, hadamard)
    kx = dequantize_rows(qz["kc"], qz["ksf"], g_k)
    vx = dequantize_rows(qz["vc"], qz["vsf"], g_v)
    T = kx.shape[0]
    if q_start is None:
        q_start = T - 1
    return attention(q, q_start, s, kx, vx, hadamard), qz
