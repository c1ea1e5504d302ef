"""Parity at the full sizes of the five workloads, in the launch configurations
the bench uses, on sampled outputs the oracle computes one by one.

Calibration is compared in full; codes and scales bit for bit on sampled
(layer, sequence) pairs; attention rows within the tolerance of
tests/harness.py, for bf16 output (the bench's) and for fp32 output at the
strict max-abs bound (the same launch with the other output type).
"""
import numpy as np
import pytest
import torch

import harness
import synth
from test_gpu_parity import assert_codes_equal

pytestmark = pytest.mark.gpu


def check_calibration(p):
    cal = harness.oracle_calibration(p)
    for got, want, name in zip(harness.calib_host(p), cal, ("s", "inv_s", "g_K", "g_V")):
        np.testing.assert_array_equal(got, want, err_msg=name)
    return cal


@pytest.mark.parametrize("name", ["qwen3_8b", "hadamard"])
def test_prefix_append_and_one_decode_step(kvq, name):
    w = synth.WORKLOADS[name]
    B = w.batch
    sample_layers = [0, w.num_layers // 2, w.num_layers - 1]
    sample_seqs = sorted({0, B // 2, B - 1})
    keep = {(l, b) for l in sample_layers for b in sample_seqs}
    p = harness.build_problem(kvq, w, lens=[w.context] * B, gen_device="cuda", keep=keep,
                              all_layers_one_call=(name == "qwen3_8b"))
    cal = check_calibration(p)
    for (li, b) in sorted(keep):
        assert_codes_equal(p, li, b, w.context, cal)
    q = torch.stack([synth.decode_queries(w, l, 0, "cuda") for l in range(w.num_layers)])
    outs = {tag: kvq.decode_attention(p.shape, p.calib, p.cache, q, p.page_table.cuda(), p.lens.cuda(),
                                      out_dtype=dt).float().cpu().numpy()
            for dt, tag in ((torch.bfloat16, "bf16"), (torch.float32, "f32"))}
    qh = q.float().cpu().numpy()
    n = w.context
    for (li, b) in sorted(keep):
        want = harness.oracle_attend(p, li, b, qh[li, b][None], n - 1, n, cal)
        for tag, out in outs.items():
            harness.check_attention(out[li, b], want[0], f"{name} layer {li} seq {b} {tag}")


def test_ragged_decode_64_steps(kvq):
    w = synth.WORKLOADS["ragged"]
    lens = synth.ragged_lengths(w)
    S = w.decode_steps
    order = torch.argsort(lens)
    sample_seqs = sorted({int(order[0]), int(order[-1]), int(order[len(order) // 2]), 5})
    sample_layers = [0, 35]
    keep = {(l, b) for l in sample_layers for b in sample_seqs}
    p = harness.build_problem(kvq, w, lens=lens, extra_tokens=S, gen_device="cuda", keep=keep, keep_tails=True)
    cal = check_calibration(p)
    tk, tv = p.tails
    pt = p.page_table.cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    pos = torch.arange(S)[:, None] + lens[None, :].long()
    slots = synth.slot_mapping(p.page_table, torch.arange(w.batch)[None, :].expand(S, -1).reshape(-1),
                               pos.reshape(-1)).view(S, w.batch).cuda()
    for s in range(S):
        kvq.quantize_append(p.shape, p.calib, p.cache, tk[s].contiguous(), tv[s].contiguous(), slots[s],
                            status=status)
        seq_lens = (lens + s + 1).to(torch.int32)
        q = torch.stack([synth.decode_queries(w, l, s, "cuda") for l in range(w.num_layers)])
        out = kvq.decode_attention(p.shape, p.calib, p.cache, q, pt, seq_lens.cuda(), out_dtype=torch.bfloat16,
                                   status=status)
        if s in (0, S // 2 - 1, S - 1):
            outs = {"bf16": out.float().cpu().numpy(),
                    "f32": kvq.decode_attention(p.shape, p.calib, p.cache, q, pt, seq_lens.cuda(),
                                                out_dtype=torch.float32, status=status).cpu().numpy()}
            qh = q.float().cpu().numpy()
            for (li, b) in sorted(keep):
                n = int(seq_lens[b])
                if s == S - 1:
                    assert_codes_equal(p, li, b, n, cal)
                want = harness.oracle_attend(p, li, b, qh[li, b][None], n - 1, n, cal)
                for tag, o in outs.items():
                    harness.check_attention(o[li, b], want[0], f"ragged step {s} layer {li} seq {b} len {n} {tag}")
    torch.cuda.synchronize()
    assert status.item() == 0


def test_chunked_prefill(kvq):
    w = synth.WORKLOADS["prefill"]
    B, Tq, P0 = w.batch, w.prefill_chunk, w.context
    sample = [(0, 0), (35, B - 1)]
    keep = set(sample)
    lens = [P0 + Tq] * B
    p = harness.build_problem(kvq, w, lens=lens, gen_device="cuda", keep=keep)
    cal = check_calibration(p)
    q = torch.stack([synth.prefill_queries(w, l, "cuda") for l in range(w.num_layers)])   # [L][B][Tq][Hq][D]
    q_start = torch.full((B,), P0, dtype=torch.int32, device="cuda")
    rows = [0, 1, 255, Tq - 1]
    outs = {}
    for dt, tag in ((torch.bfloat16, "bf16"), (torch.float32, "f32")):
        out = kvq.prefill_attention(p.shape, p.calib, p.cache, q, q_start, p.page_table.cuda(), p.lens.cuda(),
                                    out_dtype=dt)
        outs[tag] = out[:, :, rows].float().cpu().numpy()
        del out
    for (li, b) in sample:
        qh = q[li, b, rows].float().cpu().numpy()
        for r_i, r in enumerate(rows):
            want = harness.oracle_attend(p, li, b, qh[r_i][None], P0 + r, lens[b], cal)
            for tag, out_h in outs.items():
                harness.check_attention(out_h[li, b, r_i], want[0], f"prefill layer {li} seq {b} row {r} {tag}")


@pytest.mark.parametrize("variant", ["klt", "bf16_keys"])
def test_ragged_variants_full_size(kvq, variant):
    # the ragged workload (36 layers, 64 sequences of 1024..8192 tokens) with
    # the static per-head KLT (bench.py --klt) or the mixed cache of bf16 keys
    # and NVFP4 values (bench.py --k-format bf16), as the bench launches them:
    # one step appended into all 36 layers, then all 36 layers decoded.
    # Codes and scales bit for bit and attention rows within tolerance, on
    # sampled (layer, sequence) pairs.  The KLT variant runs on the oracle's
    # calibration (its eigh basis, smoothing and tensor scales written into
    # the Calibration), so the oracle reads no device value.
    w = synth.WORKLOADS["ragged"]
    lens = synth.ragged_lengths(w)
    order = torch.argsort(lens)
    sample_seqs = sorted({int(order[0]), int(order[-1]), int(order[len(order) // 2])})
    keep = {(l, b) for l in (0, 35) for b in sample_seqs}
    p = harness.build_problem(kvq, w, lens=lens, extra_tokens=1, gen_device="cuda", keep=keep, keep_tails=True,
                              klt=(variant == "klt"), k_format=(1 if variant == "bf16_keys" else 0))
    cal = harness.checked_calibration(p)
    tk, tv = p.tails
    slots = synth.slot_mapping(p.page_table, torch.arange(w.batch), lens.long()).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    kvq.quantize_append(p.shape, p.calib, p.cache, tk[0].contiguous(), tv[0].contiguous(), slots, status=status)
    seq_lens = (lens + 1).to(torch.int32)
    q = torch.stack([synth.decode_queries(w, l, 0, "cuda") for l in range(w.num_layers)])
    outs = {tag: kvq.decode_attention(p.shape, p.calib, p.cache, q, p.page_table.cuda(), seq_lens.cuda(),
                                      out_dtype=dt, status=status).float().cpu().numpy()
            for dt, tag in ((torch.bfloat16, "bf16"), (torch.float32, "f32"))}
    assert status.item() == 0
    qh = q.float().cpu().numpy()
    for (li, b) in sorted(keep):
        n = int(seq_lens[b])
        assert_codes_equal(p, li, b, n, cal)
        want = harness.oracle_attend(p, li, b, qh[li, b][None], n - 1, n, cal)
        for tag, out in outs.items():
            harness.check_attention(out[li, b], want[0], f"ragged {variant} layer {li} seq {b} len {n} {tag}")
