"""Test harness: drive the CUDA library and the oracle on the same inputs.

Inputs come from ``synth``; the oracle receives host copies of exactly the
tensors the library saw.  The cache is read back and unpacked here following
the byte layout documented in ``include/kvq.h`` (this file's own code, shared
with neither side).
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

import oracle
import synth

# ------------------------------------------------------------------ tolerances
# Attention outputs against the oracle on the same dequantised cache:
# rel-L2 <= 2e-3 and max-abs <= 1e-2 (fp32 accumulate).  With bf16 outputs the
# max-abs bound is widened to one bf16 ulp of the oracle value where that is
# larger, since rounding the output alone can exceed 1e-2 when |o| >= 4.
REL_L2 = 2e-3
MAX_ABS = 1e-2


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    a = np.abs(x).astype(np.float64)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return 2.0 ** (e - 7)


def check_attention(got, want, what=""):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape, (got.shape, want.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - want)
    rel = np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30)
    bound = np.maximum(MAX_ABS, bf16_ulp(want)) if what.endswith("bf16") else MAX_ABS
    worst = np.unravel_index(np.argmax(err - bound), err.shape)
    assert rel <= REL_L2, f"{what}: rel-L2 {rel:.3e} > {REL_L2}"
    assert np.all(err <= bound), f"{what}: max-abs {err[worst]:.3e} at {worst} (want {want[worst]:.4f})"
    return rel, float(err.max())


# ------------------------------------------------------------------ cache readback
def unpack_nibbles(b: np.ndarray) -> np.ndarray:
    """[..., 64] code bytes -> [..., 128] codes (low nibble = even element)."""
    out = np.empty(b.shape[:-1] + (2 * b.shape[-1],), np.uint8)
    out[..., 0::2] = b & 0x0F
    out[..., 1::2] = b >> 4
    return out


def read_tokens(cache_layer: np.ndarray, Hkv: int, page_table_row: np.ndarray, n: int, k_format: int = 0):
    """Codes and scales of tokens 0..n-1 of one sequence, in logical layout:
    kc, vc [n][H][128] one code per byte; ksf, vsf [n][H][8].  With bf16 keys
    (k_format 1) kc holds the key values as fp32 [n][H][128] and ksf is None."""
    t = np.arange(n)
    pages = page_table_row[t // 16]
    off = t % 16
    if k_format == 1:
        tiles = cache_layer.reshape(cache_layer.shape[0], Hkv, 5248)
        sel = tiles[pages]                               # [n][H][5248]
        kb = np.ascontiguousarray(sel[:, :, 0:4096]).view(np.uint16).reshape(n, Hkv, 16, 128)[np.arange(n), :, off]
        kx = (kb.astype(np.uint32) << 16).view(np.float32)
        vcb = sel[:, :, 4096:5120].reshape(n, Hkv, 16, 64)[np.arange(n), :, off]
        vsf = sel[:, :, 5120:5248].reshape(n, Hkv, 8, 16)[np.arange(n), :, :, off]
        return kx, None, unpack_nibbles(vcb), vsf
    tiles = cache_layer.reshape(cache_layer.shape[0], Hkv, 2304)
    sel = tiles[pages]                                   # [n][H][2304]
    kcb = sel[:, :, 0:1024].reshape(n, Hkv, 16, 64)[np.arange(n), :, off]
    ksf = sel[:, :, 1024:1152].reshape(n, Hkv, 16, 8)[np.arange(n), :, off]
    vcb = sel[:, :, 1152:2176].reshape(n, Hkv, 16, 64)[np.arange(n), :, off]
    vsf = sel[:, :, 2176:2304].reshape(n, Hkv, 8, 16)[np.arange(n), :, :, off]
    return unpack_nibbles(kcb), ksf, unpack_nibbles(vcb), vsf


# ------------------------------------------------------------------ problem setup
@dataclasses.dataclass
class Problem:
    """A workload instance on the device plus what the oracle needs."""
    w: synth.Workload
    layers: list
    lens: torch.Tensor          # [B] int32 cached tokens per sequence
    page_table: torch.Tensor    # [B][maxp] int32 (host)
    num_pages: int
    shape: object
    calib: object
    cache: object
    k_calib: np.ndarray         # [nl][W][T][H][D] fp32 host copies
    v_calib: np.ndarray
    seqs: dict                  # (layer index, b) -> (k, v) fp32 host [n][H][D]


def build_problem(kvq, w: synth.Workload, lens, layers=None, extra_tokens: int = 0, shuffle: bool = True,
                  keep_host=True, device="cuda", gen_device="cpu", keep=None, all_layers_one_call=False,
                  keep_tails=False, native=False, k_format=0, klt=False, exclude_pos0=True):
    """Calibrate, then append each sequence's first lens[b] tokens.

    keep:      optional set of (layer index, sequence) whose host copies are kept
               (all when None and keep_host).
    all_layers_one_call: append every layer with one quantize_append call
               (K/V [nl][T][Hkv][D]) instead of one call per layer.
    keep_tails: also return the extra_tokens tail of every sequence on the
               device, as tails_k/v [extra][nl][B][Hkv][D].
    native:    calibrate the keys in their native basis (no smoothing).
    k_format:  1 for the mixed cache (bf16 keys, NVFP4 values).
    klt:       smoothing plus the static per-head KLT.  The library runs on the
               oracle's own calibration (fp64 eigh basis rounded to fp32, its
               smoothing and tensor scales), written into a caller-owned
               Calibration, so no value the oracle reads comes from the
               device.  kvq_calibrate_klt itself is checked as a calibration
               in tests/test_gpu_klt.py.
    exclude_pos0: leave position 0 of every window out of the smoothing
               absmax (and of the KLT's second moment).
    """
    layers = list(range(w.num_layers)) if layers is None else list(layers)
    lens = torch.as_tensor(lens, dtype=torch.int32)
    nl, B = len(layers), len(lens)
    shape = kvq.Shape(num_layers=nl, num_q_heads=w.num_q_heads, num_kv_heads=w.num_kv_heads,
                      use_hadamard=w.hadamard, k_format=k_format, use_klt=klt)
    wins = [synth.calibration_windows(w, l, gen_device) for l in layers]
    kc = torch.stack([x[0] for x in wins])
    vc = torch.stack([x[1] for x in wins])
    del wins
    klt_cal = klt_U = None
    if klt:
        kh, vh = kc.float().cpu().numpy(), vc.float().cpu().numpy()
        s_o, inv_o, klt_U, _ = oracle.calibrate_klt(kh, vh, exclude_pos0=exclude_pos0)
        gk_o, gv_o = oracle.klt_tensor_scales(kh, vh, inv_o, klt_U)
        klt_cal = (s_o, inv_o, gk_o, gv_o)
        calib = kvq.Calibration(*(torch.from_numpy(np.ascontiguousarray(x)).to(device) for x in klt_cal),
                                k_klt=torch.from_numpy(klt_U).to(device))
    elif native:
        calib = kvq.calibrate_native(shape, kc.to(device).contiguous(), vc.to(device).contiguous())
    else:
        calib = kvq.calibrate_smoothing(shape, kc.to(device).contiguous(), vc.to(device).contiguous(),
                                        exclude_pos0=exclude_pos0)
    page_table, num_pages = synth.build_page_table(w, lens + extra_tokens, shuffle=shuffle)
    cache = kvq.new_cache(shape, num_pages, device)
    seqs = {}
    tails = None
    if keep_tails and extra_tokens:
        tails = (torch.empty(extra_tokens, nl, B, w.num_kv_heads, w.head_dim, dtype=w.dtype, device=device),
                 torch.empty(extra_tokens, nl, B, w.num_kv_heads, w.head_dim, dtype=w.dtype, device=device))
    slots = torch.cat([synth.slot_mapping(page_table, torch.full((int(n),), b), torch.arange(int(n)))
                       for b, n in enumerate(lens.tolist())]).to(device)
    layer_k, layer_v = [], []
    for li, l in enumerate(layers):
        ks, vs = [], []
        for b in range(B):
            n = int(lens[b])
            k, v = synth.sequence_kv(w, l, b, n + extra_tokens, gen_device)
            if keep_host and (keep is None or (li, b) in keep):
                seqs[(li, b)] = (k.float().cpu().numpy(), v.float().cpu().numpy())
            if tails is not None:
                tails[0][:, li, b] = k[n:].to(device)
                tails[1][:, li, b] = v[n:].to(device)
            ks.append(k[:n])
            vs.append(v[:n])
        k = torch.cat(ks).to(device)
        v = torch.cat(vs).to(device)
        del ks, vs
        if all_layers_one_call:
            layer_k.append(k)
            layer_v.append(v)
        else:
            kvq.quantize_append(shape, calib, cache, k.contiguous(), v.contiguous(), slots, layer0=li)
    if all_layers_one_call:
        kvq.quantize_append(shape, calib, cache, torch.stack(layer_k), torch.stack(layer_v), slots, layer0=0)
    p = Problem(w, layers, lens, page_table, num_pages, shape, calib, cache,
                kc.float().cpu().numpy(), vc.float().cpu().numpy(), seqs)
    p.tails = tails
    p.native = native
    p.k_format = k_format
    p.klt = klt
    p.klt_U = klt_U            # [nl][Hkv][128][128] fp32, the oracle's basis (klt only)
    p.klt_cal = klt_cal
    p.exclude_pos0 = exclude_pos0
    return p


def oracle_calibration(p: Problem):
    """The oracle's calibration of the problem: (s, inv_s, g_K, g_V)."""
    if getattr(p, "klt", False):
        return p.klt_cal
    return oracle.calibrate(p.k_calib, p.v_calib, exclude_pos0=getattr(p, "exclude_pos0", True),
                            hadamard=p.w.hadamard, smooth=not getattr(p, "native", False))


def calib_host(p: Problem):
    """The library's calibration arrays, read back from the device."""
    return (p.calib.k_smooth.cpu().numpy(), p.calib.k_inv_smooth.cpu().numpy(),
            p.calib.k_gscale.cpu().numpy(), p.calib.v_gscale.cpu().numpy())


def checked_calibration(p: Problem):
    """The oracle's calibration, after checking the library's bit for bit
    against it; every oracle comparison then runs on the oracle's values."""
    cal = oracle_calibration(p)
    for got, want, name in zip(calib_host(p), cal, ("s", "inv_s", "g_K", "g_V")):
        np.testing.assert_array_equal(got, want, err_msg=f"calibration {name}")
    return cal


def oracle_sequence(p: Problem, li: int, b: int, n: int, cal):
    """Oracle codes of tokens 0..n-1 of sequence b in layer li (with bf16
    keys: kc = the rounded key values, ksf = None)."""
    s, inv, gk, gv = cal
    k, v = p.seqs[(li, b)]
    if getattr(p, "k_format", 0) == 1:
        vc, vsf = oracle.quantize_rows(v[:n], gv[li])
        return {"kc": oracle.round_bf16(k[:n]), "ksf": None, "vc": vc, "vsf": vsf}
    if getattr(p, "klt", False):
        # smoothing, then the oracle's KLT basis in the fixed FMA order
        U = p.klt_U[li]
        y = oracle.transform_keys(k[:n], inv[li])
        yk = np.stack([oracle.klt_apply(y[:, h], U[h]) for h in range(y.shape[1])], axis=1)
        kc, ksf = oracle.quantize_rows(yk, gk[li])
        vc, vsf = oracle.quantize_rows(v[:n], gv[li])
        return {"kc": kc, "ksf": ksf, "vc": vc, "vsf": vsf}
    return oracle.quantize_kv(k[:n], v[:n], inv[li], gk[li], gv[li], p.w.hadamard)


def oracle_attend(p: Problem, li: int, b: int, q_rows: np.ndarray, q_start: int, n: int, cal):
    """Oracle attention of q_rows [Tq][Hq][D] over the first n tokens
    (cal: the oracle's calibration, oracle_calibration)."""
    s, inv, gk, gv = cal
    qz = oracle_sequence(p, li, b, n, cal)
    vx = oracle.dequantize_rows(qz["vc"], qz["vsf"], gv[li])
    if getattr(p, "k_format", 0) == 1:
        # bf16 keys: the query is used as given, the keys as stored
        return oracle.attention(q_rows, q_start, np.ones_like(s[li]), qz["kc"].astype(np.float64), vx, False)
    kx = oracle.dequantize_rows(qz["kc"], qz["ksf"], gk[li])
    if getattr(p, "klt", False):
        # the query rotated to match: q~ = U^T (q * s) per kv head, in fp64
        U = p.klt_U[li].astype(np.float64)
        G = q_rows.shape[1] // U.shape[0]
        qs = np.asarray(q_rows, np.float64) * np.repeat(np.asarray(s[li], np.float64), G, axis=0)[None]
        qt = np.einsum("thc,hci->thi", qs, np.repeat(U, G, axis=0))
        return oracle.attention(qt.astype(np.float32), q_start, np.ones_like(s[li]), kx, vx, False)
    return oracle.attention(q_rows, q_start, s[li], kx, vx, p.w.hadamard)


def oracle_attend_fp4q(p: Problem, li: int, b: int, q_rows: np.ndarray, q_start: int, n: int, cal):
    """Oracle of the FP4 Q.K prefill: the query in the keys' basis (smoothing,
    rotation or the oracle's KLT basis), quantised to NVFP4 per row by the
    oracle, dequantised exactly, then attended in fp64 against the
    dequantised cache."""
    s, inv, gk, gv = cal
    qz = oracle_sequence(p, li, b, n, cal)
    kx = oracle.dequantize_rows(qz["kc"], qz["ksf"], gk[li])
    vx = oracle.dequantize_rows(qz["vc"], qz["vsf"], gv[li])
    U = p.klt_U[li] if getattr(p, "klt", False) else None
    y = oracle.query_rows_fp4(q_rows, s[li], hadamard=bool(p.w.hadamard) and U is None, U=U)
    qx = oracle.dequantize_query(*oracle.quantize_query(y))
    return oracle.attention_x(qx, q_start, kx, vx)
