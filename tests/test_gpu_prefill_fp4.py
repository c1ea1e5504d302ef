"""Chunked causal prefill with Q.K on the block-scaled FP4 tensor cores
(kvq_prefill_attention_fp4) against the oracle.

"NVFP4 attention cache on W4A4 Qwen3-8B" (rstation.ai), setup (W4A4:
activations in NVFP4, KV cache in NVFP4); "OSFP4" (paperlayer.ai summary),
Problem bullet, sec. 1, sec. D.1 (the block quantiser).  The oracle
quantises the query with the same per-row NVFP4 quantiser (bit for bit the
kernel's decisions: both take them in IEEE fp32 in one order), dequantises it
exactly and attends in fp64; the kernel must match that within the
attention tolerance.  The distance to attention with the unquantised query
is reported as well: it is the query's 4-bit quantisation error, the price
of the FP4 product.
"""
import dataclasses

import numpy as np
import pytest
import torch

import harness
import synth

pytestmark = pytest.mark.gpu


def _small(**kw):
    return dataclasses.replace(synth.WORKLOADS["qwen3_8b"], **kw)


def _run(kvq, p, q, q_start, out_dtype):
    return kvq.prefill_attention(p.shape, p.calib, p.cache, q.cuda(), q_start.cuda(), p.page_table.cuda(),
                                 p.lens.cuda(), out_dtype=out_dtype, qk_fp4=True).float().cpu().numpy()


@pytest.mark.parametrize("variant", ["smooth", "hadamard", "klt"])
def test_fp4_prefill_ragged(kvq, variant):
    # 80 query tokens: one full pair of 32-token tiles and a ragged one;
    # keys 113 and 180 long: 2 and 3 blocks of 64 with ragged tails
    w = _small(num_layers=2, batch=2, calib_windows=4 if variant == "klt" else 1,
               calib_len=128 if variant == "klt" else 64, prefill_chunk=80, hadamard=(variant == "hadamard"))
    P0, Tq = [100, 33], 80
    lens = [n + Tq for n in P0]
    p = harness.build_problem(kvq, w, lens=lens, klt=(variant == "klt"))
    cal = harness.checked_calibration(p)
    q = torch.stack([synth.prefill_queries(w, l) for l in p.layers])        # [nl][B][Tq][Hq][D]
    q_start = torch.tensor(P0, dtype=torch.int32)
    for dt, tag in ((torch.float32, "f32"), (torch.bfloat16, "bf16")):
        out = _run(kvq, p, q, q_start, dt)
        for li in range(2):
            for b in range(2):
                want = harness.oracle_attend_fp4q(p, li, b, q[li, b].float().numpy(), P0[b], lens[b], cal)
                harness.check_attention(out[li, b], want, f"fp4 prefill {variant} layer {li} seq {b} {tag}")


def test_fp4_prefill_bf16_query_and_small_groups(kvq):
    # bf16 queries; GQA group 2 (rows of heads 2, 3 of each tile are padding)
    w = _small(num_layers=1, batch=2, num_q_heads=16, num_kv_heads=8, calib_windows=1, calib_len=64,
               prefill_chunk=40)
    P0, Tq = [7, 130], 40
    lens = [n + Tq for n in P0]
    p = harness.build_problem(kvq, w, lens=lens)
    cal = harness.checked_calibration(p)
    q = synth.prefill_queries(w, 0)[None].to(torch.bfloat16)
    out = _run(kvq, p, q, torch.tensor(P0, dtype=torch.int32), torch.float32)
    for b in range(2):
        want = harness.oracle_attend_fp4q(p, 0, b, q[0, b].float().numpy(), P0[b], lens[b], cal)
        harness.check_attention(out[0, b], want, f"fp4 prefill g2 bf16-q seq {b} f32")


def test_fp4_prefill_query_quantisation_error(kvq, capsys):
    # the kernel sits on the dequantised-query oracle; the unquantised query
    # is farther by the 4-bit quantisation error of the query
    w = _small(num_layers=2, batch=2, calib_windows=1, calib_len=64, prefill_chunk=64)
    P0, Tq = [200, 64], 64
    lens = [n + Tq for n in P0]
    p = harness.build_problem(kvq, w, lens=lens)
    cal = harness.checked_calibration(p)
    q = torch.stack([synth.prefill_queries(w, l) for l in p.layers])
    out = _run(kvq, p, q, torch.tensor(P0, dtype=torch.int32), torch.float32)
    err_q, err_x, ref = [], [], []
    for li in range(2):
        for b in range(2):
            qh = q[li, b].float().numpy()
            want_q = harness.oracle_attend_fp4q(p, li, b, qh, P0[b], lens[b], cal)
            want_x = harness.oracle_attend(p, li, b, qh, P0[b], lens[b], cal)
            err_q.append(out[li, b] - want_q)
            err_x.append(out[li, b] - want_x)
            ref.append(want_x)
    nrm = np.linalg.norm(np.stack(ref))
    rel_q = np.linalg.norm(np.stack(err_q)) / nrm
    rel_x = np.linalg.norm(np.stack(err_x)) / nrm
    with capsys.disabled():
        print(f"\nfp4 Q.K prefill: rel-L2 vs dequantised-query oracle {rel_q:.3e}, "
              f"vs unquantised-query oracle {rel_x:.3e}")
    assert rel_q < 2e-3
    assert rel_x > 5 * rel_q and rel_x < 0.5


def test_fp4_prefill_full_config_sampled(kvq):
    # the prefill workload (8 sequences of 32 query heads, 512-token chunks after 8192 cached
    # tokens, 36 layers) in the bench's launch, sampled rows against the oracle
    w = synth.WORKLOADS["prefill"]
    B, Tq, P0 = w.batch, w.prefill_chunk, w.context
    sample = [(0, 0), (35, B - 1)]
    lens = [P0 + Tq] * B
    p = harness.build_problem(kvq, w, lens=lens, gen_device="cuda", keep=set(sample))
    cal = harness.checked_calibration(p)
    q = torch.stack([synth.prefill_queries(w, l, "cuda") for l in range(w.num_layers)])
    q_start = torch.full((B,), P0, dtype=torch.int32, device="cuda")
    rows = [0, 1, 255, Tq - 1]
    outs = {}
    for dt, tag in ((torch.bfloat16, "bf16"), (torch.float32, "f32")):
        out = kvq.prefill_attention(p.shape, p.calib, p.cache, q, q_start, p.page_table.cuda(), p.lens.cuda(),
                                    out_dtype=dt, qk_fp4=True)
        outs[tag] = out[:, :, rows].float().cpu().numpy()
        del out
    for (li, b) in sample:
        qh = q[li, b, rows].float().cpu().numpy()
        for r_i, r in enumerate(rows):
            want = harness.oracle_attend_fp4q(p, li, b, qh[r_i][None], P0 + r, lens[b], cal)
            for tag, out_h in outs.items():
                harness.check_attention(out_h[li, b, r_i], want[0], f"fp4 prefill layer {li} seq {b} row {r} {tag}")


def test_fp4_prefill_edges(kvq):
    # one query; keys filling exactly two 64-key blocks; a zero-length sequence
    w = _small(num_layers=1, batch=3, calib_windows=1, calib_len=64, prefill_chunk=1)
    lens = [128, 65, 0]
    p = harness.build_problem(kvq, w, lens=[128, 65, 1])
    cal = harness.checked_calibration(p)
    q = synth.prefill_queries(w, 0)[None]                     # [1][3][1][Hq][D]
    q_start = torch.tensor([127, 64, 0], dtype=torch.int32)
    out = kvq.prefill_attention(p.shape, p.calib, p.cache, q.cuda(), q_start.cuda(), p.page_table.cuda(),
                                torch.tensor(lens, dtype=torch.int32).cuda(), out_dtype=torch.float32,
                                qk_fp4=True).cpu().numpy()
    for b in range(2):
        want = harness.oracle_attend_fp4q(p, 0, b, q[0, b].float().numpy(), int(q_start[b]), lens[b], cal)
        harness.check_attention(out[0, b], want, f"fp4 prefill edge seq {b} f32")
    assert np.all(out[0, 2] == 0)


def test_fp4_prefill_device_faults_are_flagged(kvq):
    w = _small(num_layers=1, batch=2, calib_windows=1, calib_len=64, prefill_chunk=32)
    p = harness.build_problem(kvq, w, lens=[96, 96])
    cal = harness.checked_calibration(p)
    q = synth.prefill_queries(w, 0)[None]
    q_start = torch.tensor([64, 64], dtype=torch.int32)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    pt = p.page_table.clone()
    pt[1, 2] = p.num_pages + 3                                 # outside the pool
    out = kvq.prefill_attention(p.shape, p.calib, p.cache, q.cuda(), q_start.cuda(), pt.cuda(), p.lens.cuda(),
                                out_dtype=torch.float32, status=status, qk_fp4=True)
    torch.cuda.synchronize()
    assert status.item() & kvq.DEV_BAD_PAGE
    out = out.cpu().numpy()
    assert np.all(out[0, 1] == 0)
    want = harness.oracle_attend_fp4q(p, 0, 0, q[0, 0].float().numpy(), 64, 96, cal)
    harness.check_attention(out[0, 0], want, "fp4 prefill beside a bad page f32")
