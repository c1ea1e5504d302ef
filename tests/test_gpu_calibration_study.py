"""Calibration ablations of the key cache, measured through the library.

"NVFP4 attention cache on W4A4 Qwen3-8B" (rstation.ai), results table rows
"NVFP4 K only, native basis", "K: static per-channel smoothing, sqrt(absmax)
from 4 C4 windows, position 0 excluded", "K: same smoothing, but sink token
included in the absmax", "K: Hadamard-128 on head_dim", "K: Hadamard-128 +
smoothing", "K: static KLT + smoothing" and "NVFP4 V only" (bf16 keys), with observation 2 (calibrate without the sink).  The pages score
these rows by perplexity of a trained model; with synthetic inputs the score
here is the attention output error of one decode step: relative L2 norm of
(NVFP4-cache attention - exact fp64 attention on the unquantised bf16 cache)
over every (layer, sequence, query head), plus its largest per-head value.
The calibration windows are the workload's seeded synthetic windows (sink at
position 0 of each), and the window count is varied as well.

The synthetic logits have a standard deviation of 4 to 10 (outlier channels
x20), so the softmax is peaked and 4-bit keys move it visibly: the errors
are of order 0.2, far above the kernel-versus-oracle tolerance, which
compares both on the same dequantised cache.  Only orderings with a wide
margin, and that the pages' table shows as well, are asserted: smoothing
beats the native basis, and the rotation without smoothing is worse than the
native basis.
"""
import dataclasses

import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

LAYERS = (0, 1, 2, 3)


def _workload(hadamard=False, windows=4):
    return dataclasses.replace(synth.WORKLOADS["qwen3_8b"], num_layers=len(LAYERS), hadamard=hadamard,
                               calib_windows=windows)


def _sequences(w):
    """Post-RoPE K, V [n][Hkv][D] (device, bf16) of every (layer, sequence)."""
    return {(l, b): synth.sequence_kv(w, l, b, w.context, "cuda") for l in LAYERS for b in range(w.batch)}


def _reference(w, kv, q):
    """Exact softmax attention in fp64 on the unquantised cache: [nl][B][Hq][D]."""
    G = w.num_q_heads // w.num_kv_heads
    out = torch.empty(len(LAYERS), w.batch, w.num_q_heads, w.head_dim, dtype=torch.float64, device="cuda")
    for li, l in enumerate(LAYERS):
        for b in range(w.batch):
            k, v = (x.double() for x in kv[(l, b)])
            for h in range(w.num_kv_heads):
                qh = q[li, b, h * G:(h + 1) * G].double()
                p = torch.softmax(qh @ k[:, h].T / w.head_dim ** 0.5, dim=-1)
                out[li, b, h * G:(h + 1) * G] = p @ v[:, h]
    return out


def _run(kvq, w, kv, q, mode):
    """Calibrate (mode: 'excl' sink left out, 'incl' sink in, 'native' no
    smoothing, 'bf16k' bf16 keys with packed values, 'klt' smoothing then the
    static per-head KLT), append every sequence, decode one step;
    [nl][B][Hq][D] fp32."""
    shape = kvq.Shape(len(LAYERS), w.num_q_heads, w.num_kv_heads, use_hadamard=w.hadamard,
                      k_format=kvq.K_BF16 if mode == "bf16k" else kvq.K_NVFP4, use_klt=(mode == "klt"))
    win = [synth.calibration_windows(w, l, "cuda") for l in LAYERS]
    kc = torch.stack([x[0] for x in win]).contiguous()
    vc = torch.stack([x[1] for x in win]).contiguous()
    if mode == "klt":
        calib = kvq.calibrate_klt(shape, kc, vc)
    elif mode in ("native", "bf16k"):
        calib = kvq.calibrate_native(shape, kc, vc)
    else:
        calib = kvq.calibrate_smoothing(shape, kc, vc, exclude_pos0=(mode == "excl"))
    lens = torch.full((w.batch,), w.context, dtype=torch.int32)
    page_table, num_pages = synth.build_page_table(w, lens)
    cache = kvq.new_cache(shape, num_pages, "cuda")
    slots = torch.cat([synth.slot_mapping(page_table, torch.full((w.context,), b), torch.arange(w.context))
                       for b in range(w.batch)]).cuda()
    for li, l in enumerate(LAYERS):
        k = torch.cat([kv[(l, b)][0] for b in range(w.batch)])
        v = torch.cat([kv[(l, b)][1] for b in range(w.batch)])
        kvq.quantize_append(shape, calib, cache, k, v, slots, layer0=li)
    return kvq.decode_attention(shape, calib, cache, q, page_table.cuda(), lens.cuda(), out_dtype=torch.float32)


def _errors(out, ref):
    d = out.double() - ref
    rel = (d.norm() / ref.norm()).item()
    per_head = (d.norm(dim=-1) / ref.norm(dim=-1).clamp_min(1e-30)).max().item()
    return rel, per_head


def test_calibration_ablations(kvq, capsys):
    base = _workload()
    kv = _sequences(base)
    q = torch.stack([synth.decode_queries(base, l, 0, "cuda") for l in LAYERS]).contiguous()
    ref = _reference(base, kv, q)
    rows = []
    for name, w, mode in (
            ("smoothing, position 0 excluded, 4 windows", base, "excl"),
            ("smoothing, position 0 excluded, 1 window", _workload(windows=1), "excl"),
            ("smoothing, position 0 excluded, 2 windows", _workload(windows=2), "excl"),
            ("smoothing, position 0 excluded, 8 windows", _workload(windows=8), "excl"),
            ("smoothing, sink included, 4 windows", base, "incl"),
            ("native basis (no smoothing)", base, "native"),
            ("Hadamard-128 + smoothing", _workload(hadamard=True), "excl"),
            ("Hadamard-128 alone", _workload(hadamard=True), "native"),
            ("static KLT + smoothing", base, "klt"),
            ("bf16 keys, NVFP4 values", base, "bf16k")):
        rows.append((name,) + _errors(_run(kvq, w, kv, q, mode), ref))
    with capsys.disabled():
        print("\nkey calibration ablation (qwen3_8b shapes, 4 layers x 4 sequences x 2304 tokens)")
        print(f"{'variant':46s} {'rel-L2':>9s} {'worst head':>11s}")
        for name, rel, worst in rows:
            print(f"{name:46s} {rel:9.5f} {worst:11.5f}")
    err = {name: rel for name, rel, _ in rows}
    for name, rel, worst in rows:
        assert 0.0 < rel < 1.0 and worst < 10.0, (name, rel, worst)
    smooth, native = err["smoothing, position 0 excluded, 4 windows"], err["native basis (no smoothing)"]
    # table rows "NVFP4 K only, native basis" and "K: static per-channel
    # smoothing": smoothing brings the keys closer to lossless
    assert smooth < 0.9 * native
    # rows "NVFP4 K only, native basis" and "K: Hadamard-128 on head_dim": the
    # rotation alone is worse than the native basis
    assert err["Hadamard-128 alone"] > 1.1 * native
    # row "NVFP4 V only": the keys carry the gap; packed values alone cost far less
    assert err["bf16 keys, NVFP4 values"] < 0.5 * smooth
