"""Host-side checks of the C ABI: symbols, sizes, status codes, validation.

No kernel runs here; every call below either needs no device or is rejected
by host validation before any launch.
"""
import ctypes
import re

import pytest

from conftest import ROOT, read_golden


def header_functions():
    with open(f"{ROOT}/include/kvq.h") as f:
        text = f.read()
    return sorted(set(re.findall(r"^[a-z_ ]*?\**\s*(kvq_[a-z0-9_]+)\(", text, flags=re.M)))


def test_every_declared_function_is_exported(kvq_lib):
    names = header_functions()
    assert len(names) >= 11
    for n in names:
        assert hasattr(kvq_lib._lib, n), n
    assert set(names) == set(kvq_lib.EXPORTED)


def test_version_and_status_strings(kvq_lib):
    assert "sm_100a" in kvq_lib.version()
    assert kvq_lib.status_string(0) == "ok"
    assert kvq_lib.status_string(4) == "workspace too small"
    assert kvq_lib.status_string(99) == "unknown status"


def test_page_bytes(kvq_lib):
    assert kvq_lib.page_bytes(kvq_lib.Shape(36, 32, 8)) == 8 * 2304
    bad = kvq_lib.Shape(36, 32, 8, head_dim=64)
    assert kvq_lib._lib.kvq_page_bytes(ctypes.byref(bad.c())) == 0


def test_layout_sizes_against_page_one_figures(kvq_lib):
    g = {k: float(v) for k, v in read_golden("cache_sizes.txt")}
    L, H, D = int(g["num_layers"]), int(g["num_kv_heads"]), int(g["head_dim"])
    bf16_per_token = L * 2 * H * D * 2
    assert bf16_per_token == g["bf16_kib_per_token"] * 1024
    assert abs(bf16_per_token * 4 * 2304 / 1e9 - g["bf16_gb_batch4_2p3k"]) < 0.1
    per_token_layer = kvq_lib.page_bytes(kvq_lib.Shape(L, 32, H)) // 16
    assert per_token_layer == 1152                 # 2 x 8 x (64 B codes + 8 B scales)
    assert per_token_layer * L / 1024 == 40.5      # KiB per token over 36 layers
    assert bf16_per_token / (per_token_layer * L) == pytest.approx(3.5556, rel=1e-4)


def _call_decode(kvq, shape, **over):
    args = dict(calib=kvq._Calib(16, 16, 16, 16), cache=kvq._Cache(4096, 8 * 2304 * 4, 4),
                layer0=0, nlayers=1, q=256, q_dtype=1, page_table=512, maxp=64, seq_lens=768, batch=2,
                out=1024, out_dtype=1, ws=2048, ws_bytes=1 << 30, status=None)
    args.update(over)
    return kvq._lib.kvq_decode_attention(
        ctypes.byref(shape.c()) if shape is not None else None, ctypes.byref(args["calib"]),
        ctypes.byref(args["cache"]), args["layer0"], args["nlayers"], args["q"], args["q_dtype"],
        args["page_table"], args["maxp"], args["seq_lens"], args["batch"], args["out"], args["out_dtype"],
        args["ws"], args["ws_bytes"], args["status"], None)


def test_host_validation_rejects_before_launch(kvq_lib):
    kvq = kvq_lib
    s = kvq.Shape(2, 32, 8)
    assert _call_decode(kvq, None) == kvq.KVQ_EINVAL
    assert _call_decode(kvq, kvq.Shape(2, 32, 8, head_dim=64)) == kvq.KVQ_EUNSUPPORTED
    assert _call_decode(kvq, kvq.Shape(2, 32, 8, page_size=32)) == kvq.KVQ_EUNSUPPORTED
    assert _call_decode(kvq, kvq.Shape(2, 30, 8)) == kvq.KVQ_EINVAL          # Hq % Hkv
    assert _call_decode(kvq, kvq.Shape(2, 32, 3, use_hadamard=True)) != kvq.KVQ_OK
    assert _call_decode(kvq, s, q=None) == kvq.KVQ_EINVAL
    assert _call_decode(kvq, s, q=258) == kvq.KVQ_EINVAL                    # misaligned
    assert _call_decode(kvq, s, layer0=1, nlayers=2) == kvq.KVQ_EINVAL      # beyond L
    assert _call_decode(kvq, s, q_dtype=7) == kvq.KVQ_EINVAL
    assert _call_decode(kvq, s, cache=kvq._Cache(4096, 100, 4)) == kvq.KVQ_EINVAL   # stride too small
    assert _call_decode(kvq, s, cache=kvq._Cache(4100, 8 * 2304 * 4, 4)) == kvq.KVQ_EINVAL
    assert _call_decode(kvq, s, calib=kvq._Calib(16, None, 16, 16)) == kvq.KVQ_EINVAL
    need = kvq.decode_workspace_bytes(s, 1, 2, 64)
    assert need > 0
    assert _call_decode(kvq, s, ws=None) == kvq.KVQ_EWORKSPACE
    assert _call_decode(kvq, s, ws_bytes=need - 1) == kvq.KVQ_EWORKSPACE


def test_selftest_validation(kvq_lib):
    kvq = kvq_lib
    f = kvq._lib.kvq_selftest_wait_timeout
    assert f(None, 1_000_000, None) == kvq.KVQ_EINVAL
    assert f(256, 10, None) == kvq.KVQ_EINVAL                   # limit below 1 us
    assert f(256, 10 ** 12, None) == kvq.KVQ_EINVAL             # limit above 10 s


def test_append_validation(kvq_lib):
    kvq = kvq_lib
    s = kvq.Shape(1, 32, 8)
    cal, cache = kvq._Calib(16, 16, 16, 16), kvq._Cache(4096, 8 * 2304 * 4, 4)
    f = kvq._lib.kvq_quantize_append
    # zero tokens: nothing to do, no device needed
    assert f(ctypes.byref(s.c()), ctypes.byref(cal), ctypes.byref(cache), 0, 1, None, None, 1, None, 0,
             None, None) == kvq.KVQ_OK
    assert f(ctypes.byref(s.c()), ctypes.byref(cal), ctypes.byref(cache), 0, 1, None, 256, 1, 512, 4,
             None, None) == kvq.KVQ_EINVAL
    assert f(ctypes.byref(s.c()), ctypes.byref(cal), ctypes.byref(cache), 0, 1, 256, 256, 1, 516, 4,
             None, None) == kvq.KVQ_EINVAL                                  # slots misaligned
    assert f(ctypes.byref(s.c()), ctypes.byref(cal), ctypes.byref(cache), 0, 1, 256, 256, 1, 512, -1,
             None, None) == kvq.KVQ_EINVAL


def test_decode_split_plan_is_deterministic(kvq_lib):
    kvq = kvq_lib
    s = kvq.Shape(36, 32, 8)
    # many (layer, sequence, kv head) units: no split and no workspace
    assert kvq.decode_workspace_bytes(s, 36, 64, 516) == 0
    # few units with long sequences: split-K partials need a workspace
    a = kvq.decode_workspace_bytes(kvq.Shape(1, 32, 8), 1, 1, 512)
    assert a > 0 and a == kvq.decode_workspace_bytes(kvq.Shape(1, 32, 8), 1, 1, 512)


def test_workspace_layout(kvq_lib):
    # a workspace starts with the split merge's 4096-byte counter header, then
    # the partials [nl][B][Hq][splits][132] fp32 (256-byte aligned), then with
    # a KLT cache the rotated queries [nl][B][Hq][128] fp32; the prefill's
    # rotated queries also start after the header
    kvq = kvq_lib
    s = kvq.Shape(1, 32, 8)
    ws = kvq.decode_workspace_bytes(s, 1, 1, 512)
    splits = (ws - 4096) // (32 * 132 * 4)
    assert ws == 4096 + 32 * splits * 132 * 4 and splits > 1
    klt = kvq.Shape(1, 32, 8, use_klt=True)
    part = 32 * splits * 132 * 4
    assert kvq.decode_workspace_bytes(klt, 1, 1, 512) == 4096 + (part + 255) // 256 * 256 + 32 * 128 * 4
    # no split, no KLT: no workspace; no split with a KLT cache: header + queries
    assert kvq.decode_workspace_bytes(kvq.Shape(36, 32, 8), 36, 64, 516) == 0
    assert kvq.decode_workspace_bytes(kvq.Shape(36, 32, 8, use_klt=True), 36, 64, 516) == 4096 + 36 * 64 * 32 * 128 * 4
    assert kvq.prefill_workspace_bytes(kvq.Shape(2, 32, 8), 2, 8, 512) == 0
    assert kvq.prefill_workspace_bytes(kvq.Shape(2, 32, 8, use_klt=True), 2, 8, 512) == 4096 + 2 * 8 * 512 * 32 * 128 * 4
    # the binding's workspaces are zero-filled
    w = kvq.new_workspace(64, "cpu")
    assert w.dtype.itemsize == 1 and int(w.sum()) == 0


def test_mixed_cache_key_format_validation(kvq_lib):
    kvq = kvq_lib
    bf = kvq.Shape(2, 32, 8, k_format=kvq.K_BF16)
    assert kvq.page_bytes(bf) == 8 * 5248
    assert _call_decode(kvq, kvq.Shape(2, 32, 8, k_format=2)) == kvq.KVQ_EINVAL
    # bf16 keys are stored untransformed: no rotation
    assert _call_decode(kvq, kvq.Shape(2, 32, 8, use_hadamard=True, k_format=kvq.K_BF16)) == kvq.KVQ_EINVAL
    # a layer stride sized for packed keys is too small for bf16 keys
    assert _call_decode(kvq, bf, cache=kvq._Cache(4096, 8 * 2304 * 4, 4)) == kvq.KVQ_EINVAL
    # the prefill checks the cache against the bf16-key tile size too
    st = kvq._lib.kvq_prefill_attention(
        ctypes.byref(bf.c()), ctypes.byref(kvq._Calib(16, 16, 16, 16)), ctypes.byref(kvq._Cache(4096, 8 * 2304 * 4, 4)),
        0, 1, 256, 1, 8, 512, 768, 64, 1024, 2, 2048, 1, None, 0, None, None)
    assert st == kvq.KVQ_EINVAL


def test_fp4_prefill_needs_packed_keys(kvq_lib):
    # FP4 Q.K reads the keys' E2M1 codes: a bf16-key (mixed) cache is refused
    kvq = kvq_lib
    bf = kvq.Shape(2, 32, 8, k_format=kvq.K_BF16)
    args = (ctypes.byref(kvq._Calib(16, 16, 16, 16)), ctypes.byref(kvq._Cache(4096, 8 * 5248 * 4, 4)),
            0, 1, 256, 1, 8, 512, 768, 64, 1024, 2, 2048, 1, None, 0, None, None)
    assert kvq._lib.kvq_prefill_attention_fp4(ctypes.byref(bf.c()), *args) == kvq.KVQ_EINVAL
    # the same arguments pass kvq_prefill_attention's checks (and stop at the device check here)
    assert kvq._lib.kvq_prefill_attention(ctypes.byref(bf.c()), *args) != kvq.KVQ_EINVAL
    # packed keys pass the FP4 call's checks too
    pk = kvq.Shape(2, 32, 8)
    args = (ctypes.byref(kvq._Calib(16, 16, 16, 16)), ctypes.byref(kvq._Cache(4096, 8 * 2304 * 4, 4)),
            0, 1, 256, 1, 8, 512, 768, 64, 1024, 2, 2048, 1, None, 0, None, None)
    assert kvq._lib.kvq_prefill_attention_fp4(ctypes.byref(pk.c()), *args) != kvq.KVQ_EINVAL
