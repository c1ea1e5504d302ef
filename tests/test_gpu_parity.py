"""Parity of the CUDA path with the oracle on small workloads.

Codes and scales must match bit for bit; attention outputs within the
tolerance stated in tests/harness.py.
"""
import dataclasses

import numpy as np
import pytest
import torch

import harness
import oracle
import synth

pytestmark = pytest.mark.gpu


def small(name="qwen3_8b", **kw):
    return dataclasses.replace(synth.WORKLOADS[name], **kw)


def assert_codes_equal(p, li, b, n, cal):
    layer = p.cache.data[li].cpu().numpy()
    kc, ksf, vc, vsf = harness.read_tokens(layer, p.w.num_kv_heads, p.page_table[b].numpy(), n,
                                           getattr(p, "k_format", 0))
    ref = harness.oracle_sequence(p, li, b, n, cal)
    for name, got in (("kc", kc), ("ksf", ksf), ("vc", vc), ("vsf", vsf)):
        want = ref[name]
        if want is None:
            assert got is None
            continue
        if not np.array_equal(got, want):
            idx = np.argwhere(got != want)[0]
            raise AssertionError(f"{name} mismatch layer {li} seq {b} at {tuple(idx)}: "
                                 f"device {got[tuple(idx)]} oracle {want[tuple(idx)]} ({(got != want).sum()} total)")


def decode_all(kvq, p, step=0, out_dtype=torch.float32, lens=None):
    q = torch.stack([synth.decode_queries(p.w, l, step) for l in p.layers])
    lens = p.lens if lens is None else lens
    out = kvq.decode_attention(p.shape, p.calib, p.cache, q.cuda(), p.page_table.cuda(), lens.cuda(),
                               out_dtype=out_dtype)
    return q.float().numpy(), out.float().cpu().numpy()


def test_tiny_workload_end_to_end(kvq):
    w = synth.WORKLOADS["tiny"]
    p = harness.build_problem(kvq, w, lens=[256])
    cal = harness.oracle_calibration(p)
    for got, want, name in zip(harness.calib_host(p), cal, ("s", "inv_s", "g_K", "g_V")):
        np.testing.assert_array_equal(got, want, err_msg=name)
    assert_codes_equal(p, 0, 0, 256, cal)
    for dt, tag in ((torch.float32, "f32"), (torch.bfloat16, "bf16")):
        q, out = decode_all(kvq, p, out_dtype=dt)
        want = harness.oracle_attend(p, 0, 0, q[0, 0][None], 255, 256, cal)
        harness.check_attention(out[0, 0], want[0], f"tiny decode {tag}")


@pytest.mark.parametrize("hadamard", [False, True])
def test_ragged_multilayer_bf16(kvq, hadamard):
    w = small(num_layers=3, batch=4, calib_windows=2, calib_len=64, hadamard=hadamard)
    lens = [1, 17, 300, 129]
    p = harness.build_problem(kvq, w, lens=lens, layers=[0, 2])
    cal = harness.oracle_calibration(p)
    for got, want in zip(harness.calib_host(p), cal):
        np.testing.assert_array_equal(got, want)
    for li in range(2):
        for b, n in enumerate(lens):
            assert_codes_equal(p, li, b, n, cal)
    for dt, tag in ((torch.float32, "f32"), (torch.bfloat16, "bf16")):
        q, out = decode_all(kvq, p, out_dtype=dt)
        for li in range(2):
            for b, n in enumerate(lens):
                want = harness.oracle_attend(p, li, b, q[li, b][None], n - 1, n, cal)
                harness.check_attention(out[li, b], want[0], f"layer {li} seq {b} len {n} {tag}")


@pytest.mark.parametrize("hadamard", [False, True])
def test_native_basis_keys(kvq, hadamard):
    # "NVFP4 attention cache on W4A4 Qwen3-8B", results table row "NVFP4 K
    # only, native basis": no smoothing
    w = small(num_layers=2, batch=3, calib_windows=2, calib_len=64, hadamard=hadamard)
    lens = [5, 140, 301]
    p = harness.build_problem(kvq, w, lens=lens, native=True)
    cal = harness.oracle_calibration(p)
    assert np.all(cal[0] == 1)
    for got, want, name in zip(harness.calib_host(p), cal, ("s", "inv_s", "g_K", "g_V")):
        np.testing.assert_array_equal(got, want, err_msg=name)
    for li in range(2):
        for b, n in enumerate(lens):
            assert_codes_equal(p, li, b, n, cal)
    q, out = decode_all(kvq, p)
    for li in range(2):
        for b, n in enumerate(lens):
            want = harness.oracle_attend(p, li, b, q[li, b][None], n - 1, n, cal)
            harness.check_attention(out[li, b], want[0], f"native layer {li} seq {b} len {n}")


@pytest.mark.parametrize("hadamard", [False, True])
def test_sink_included_smoothing(kvq, hadamard):
    # "NVFP4 attention cache on W4A4 Qwen3-8B", results table row "K: same
    # smoothing, but sink token included in the absmax" (observation 2):
    # kvq_calibrate_smoothing with exclude_pos0 = 0, then append and decode
    w = small(num_layers=2, batch=3, calib_windows=2, calib_len=64, hadamard=hadamard)
    lens = [9, 140, 301]
    p = harness.build_problem(kvq, w, lens=lens, exclude_pos0=False)
    cal = harness.checked_calibration(p)
    # the sink (x40) now sets the absmax of its channels
    s_ex = oracle.calibrate(p.k_calib, p.v_calib, exclude_pos0=True, hadamard=hadamard)[0]
    assert np.all(cal[0] >= s_ex) and np.any(cal[0] > s_ex)
    for li in range(2):
        for b, n in enumerate(lens):
            assert_codes_equal(p, li, b, n, cal)
    for dt, tag in ((torch.float32, "f32"), (torch.bfloat16, "bf16")):
        q, out = decode_all(kvq, p, out_dtype=dt)
        for li in range(2):
            for b, n in enumerate(lens):
                want = harness.oracle_attend(p, li, b, q[li, b][None], n - 1, n, cal)
                harness.check_attention(out[li, b], want[0], f"sink-included layer {li} seq {b} {tag}")


@pytest.mark.parametrize("name", ["tiny", "qwen3_8b"])
def test_mixed_cache_bf16_keys(kvq, name):
    # "NVFP4 attention cache on W4A4 Qwen3-8B", results table row "NVFP4 V
    # only": bf16 keys (bit-exact: copied, or rounded from fp32), NVFP4 values
    if name == "tiny":
        w, lens, layers = synth.WORKLOADS["tiny"], [256], [0]
    else:
        w, lens, layers = small(num_layers=2, batch=3, calib_windows=1, calib_len=64), [7, 160, 333], [0, 1]
    p = harness.build_problem(kvq, w, lens=lens, layers=layers, k_format=1)
    cal = harness.oracle_calibration(p)
    for li in range(len(layers)):
        for b, n in enumerate(lens):
            assert_codes_equal(p, li, b, n, cal)
    for dt, tag in ((torch.float32, "f32"), (torch.bfloat16, "bf16")):
        q, out = decode_all(kvq, p, out_dtype=dt)
        for li in range(len(layers)):
            for b, n in enumerate(lens):
                want = harness.oracle_attend(p, li, b, q[li, b][None], n - 1, n, cal)
                harness.check_attention(out[li, b], want[0], f"bf16-key layer {li} seq {b} len {n} {tag}")


def test_many_units_single_split(kvq):
    # enough (layer, sequence, head) units that the decode needs no split
    w = small(num_layers=10, batch=64, calib_windows=1, calib_len=32)
    lens = (torch.arange(64) % 7 * 9 + 1).tolist()
    p = harness.build_problem(kvq, w, lens=lens)
    assert kvq.decode_workspace_bytes(p.shape, 10, 64, p.page_table.shape[1]) == 0
    cal = harness.oracle_calibration(p)
    q, out = decode_all(kvq, p, out_dtype=torch.bfloat16)
    for li in (0, 9):
        for b in (0, 5, 63):
            n = lens[b]
            want = harness.oracle_attend(p, li, b, q[li, b][None], n - 1, n, cal)
            harness.check_attention(out[li, b], want[0], f"layer {li} seq {b} bf16")


def test_split_batch_edge_lengths_and_a_bad_page(kvq):
    # 2 layers x 64 sequences = 128 (layer, sequence) units, too few to fill
    # the GPU unsplit: a split decode.  Lengths include 0, one token, a full
    # page and one past it; a bad page id poisons one sequence only, in both
    # layers, and leaves the others within tolerance.
    w = small(num_layers=2, batch=64, calib_windows=1, calib_len=64)
    lens = [0, 1, 16, 17] + [(37 * b) % 600 + 2 for b in range(4, 64)]
    p = harness.build_problem(kvq, w, lens=lens)
    assert kvq.decode_workspace_bytes(p.shape, 2, 64, p.page_table.shape[1]) > 0     # split
    cal = harness.oracle_calibration(p)
    bad = 5
    pt = p.page_table.clone()
    pt[bad, 1] = p.num_pages + 5
    q = torch.stack([synth.decode_queries(w, l, 0) for l in p.layers])
    for dt, tag in ((torch.float32, "f32"), (torch.bfloat16, "bf16")):
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        out = kvq.decode_attention(p.shape, p.calib, p.cache, q.cuda(), pt.cuda(), p.lens.cuda(), status=status,
                                   out_dtype=dt).float().cpu().numpy()
        torch.cuda.synchronize()
        assert status.item() & kvq.DEV_BAD_PAGE
        assert np.all(out[:, bad] == 0) and np.all(out[:, 0] == 0)
        for li in (0, 1):
            for b in (1, 2, 3, 4, 17, 63):
                n = lens[b]
                want = harness.oracle_attend(p, li, b, q[li, b].float().numpy()[None], n - 1, n, cal)
                harness.check_attention(out[li, b], want[0], f"split batch, layer {li} seq {b} {tag}")


def test_long_sequence_many_splits(kvq):
    w = small(num_layers=1, batch=1, calib_windows=1, calib_len=128)
    p = harness.build_problem(kvq, w, lens=[5000])
    assert kvq.decode_workspace_bytes(p.shape, 1, 1, p.page_table.shape[1]) > 0
    cal = harness.oracle_calibration(p)
    q, out = decode_all(kvq, p)
    want = harness.oracle_attend(p, 0, 0, q[0, 0][None], 4999, 5000, cal)
    harness.check_attention(out[0, 0], want[0], "5000 tokens f32")


def test_split_merge_counters_and_workspace_reuse(kvq):
    # The fused split merge keeps one arrival counter per (layer, sequence) in
    # the first 4096 bytes of the workspace: zero before the first call, left
    # zero by every call.  One zero-filled workspace then serves split decodes
    # of different shapes in any order, bit for bit like fresh workspaces; a
    # header that was not zero-filled is reported (KVQ_DEV_BAD_WORKSPACE), not
    # trapped.
    w = small(num_layers=2, batch=3, calib_windows=1, calib_len=64)
    pa = harness.build_problem(kvq, w, lens=[3000, 45, 700])
    pb = harness.build_problem(kvq, small(num_layers=1, batch=1, calib_windows=1, calib_len=64), lens=[5000])
    qa = torch.stack([synth.decode_queries(pa.w, l, 0) for l in pa.layers]).cuda()
    qb = torch.stack([synth.decode_queries(pb.w, l, 0) for l in pb.layers]).cuda()
    need = [kvq.decode_workspace_bytes(p.shape, len(p.layers), len(p.lens), p.page_table.shape[1]) for p in (pa, pb)]
    assert min(need) > 4096
    shared = kvq.new_workspace(max(need))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")

    def run(p, q, ws):
        return kvq.decode_attention(p.shape, p.calib, p.cache, q, p.page_table.cuda(), p.lens.cuda(),
                                    out_dtype=torch.float32, workspace=ws, status=status)

    ref_a = run(pa, qa, kvq.new_workspace(need[0]))
    ref_b = run(pb, qb, kvq.new_workspace(need[1]))
    for p, q, ref in ((pa, qa, ref_a), (pb, qb, ref_b), (pa, qa, ref_a), (pb, qb, ref_b)):
        assert torch.equal(run(p, q, shared), ref)
    torch.cuda.synchronize()
    assert status.item() == 0
    assert torch.count_nonzero(shared[:4096]).item() == 0          # the counters are back to zero
    cal = harness.oracle_calibration(pa)
    qh = qa.float().cpu().numpy()
    for li in range(2):
        for b, n in enumerate(pa.lens.tolist()):
            want = harness.oracle_attend(pa, li, b, qh[li, b][None], n - 1, n, cal)
            harness.check_attention(ref_a[li, b].cpu().numpy(), want[0], f"reused workspace layer {li} seq {b}")
    # a header that was not zero-filled: flagged
    bad = torch.full((need[0],), 0x7F, dtype=torch.uint8, device="cuda")
    run(pa, qa, bad)
    torch.cuda.synchronize()
    assert status.item() & kvq.DEV_BAD_WORKSPACE


@pytest.mark.parametrize("scale", [1.0 / 64, 3.0])
def test_flat_and_peaked_softmax(kvq, scale):
    # The decode keeps a lazy softmax reference that moves only when a score
    # passes it by more than 8 (log2 units).  A near-uniform softmax (queries
    # x 1/64: the reference never moves after the first page) and a peaked
    # one (x 3: it moves often, by large steps) both match the oracle, on a
    # split sequence (partials merged by the combine) and on unsplit ones.
    w = small(num_layers=2, batch=3, calib_windows=1, calib_len=64)
    lens = [3000, 45, 700]
    p = harness.build_problem(kvq, w, lens=lens)
    cal = harness.oracle_calibration(p)
    q = torch.stack([synth.decode_queries(w, l, 0) for l in p.layers]).float() * scale
    out = kvq.decode_attention(p.shape, p.calib, p.cache, q.cuda(), p.page_table.cuda(), p.lens.cuda(),
                               out_dtype=torch.float32).cpu().numpy()
    qh = q.numpy()
    for li in range(2):
        for b, n in enumerate(lens):
            want = harness.oracle_attend(p, li, b, qh[li, b][None], n - 1, n, cal)
            harness.check_attention(out[li, b], want[0], f"query x {scale} layer {li} seq {b}")


def test_page_order_does_not_change_results(kvq):
    w = small(num_layers=1, batch=3, calib_windows=1, calib_len=64)
    lens = [40, 200, 77]
    a = harness.build_problem(kvq, w, lens=lens, shuffle=True)
    b = harness.build_problem(kvq, w, lens=lens, shuffle=False)
    _, oa = decode_all(kvq, a)
    _, ob = decode_all(kvq, b)
    np.testing.assert_array_equal(oa, ob)


@pytest.mark.parametrize("k_format", [0, 1])
def test_prefill_chunk(kvq, k_format):
    # k_format 1: the mixed cache (bf16 keys copied into the key tile, bf16 Q.K)
    w = small(num_layers=2, batch=2, calib_windows=1, calib_len=64, prefill_chunk=48)
    P0 = [100, 33]
    Tq = 48
    lens = [n + Tq for n in P0]
    p = harness.build_problem(kvq, w, lens=lens, k_format=k_format)
    cal = harness.oracle_calibration(p)
    q = torch.stack([synth.prefill_queries(w, l) for l in p.layers])        # [nl][B][Tq][Hq][D]
    q_start = torch.tensor(P0, dtype=torch.int32)
    for dt, tag in ((torch.float32, "f32"), (torch.bfloat16, "bf16")):
        out = kvq.prefill_attention(p.shape, p.calib, p.cache, q.cuda(), q_start.cuda(), p.page_table.cuda(),
                                    p.lens.cuda(), out_dtype=dt).float().cpu().numpy()
        for li in range(2):
            for b in range(2):
                want = harness.oracle_attend(p, li, b, q[li, b].float().numpy(), P0[b], lens[b], cal)
                harness.check_attention(out[li, b], want, f"prefill k_format {k_format} layer {li} seq {b} {tag}")


def test_zero_length_gives_zero_rows(kvq):
    w = small(num_layers=1, batch=2, calib_windows=1, calib_len=32)
    p = harness.build_problem(kvq, w, lens=[20, 20])
    _, out = decode_all(kvq, p, lens=torch.tensor([0, 20], dtype=torch.int32))
    assert np.all(out[0, 0] == 0) and np.any(out[0, 1] != 0)


def test_device_faults_are_flagged_not_trapped(kvq):
    w = small(num_layers=1, batch=2, calib_windows=1, calib_len=32)
    p = harness.build_problem(kvq, w, lens=[40, 40])
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    # a page id outside the pool: the row is zeroed and BAD_PAGE set
    pt = p.page_table.clone()
    pt[1, 1] = p.num_pages + 5
    q = synth.decode_queries(w, 0, 0)[None].cuda()
    out = kvq.decode_attention(p.shape, p.calib, p.cache, q, pt.cuda(), p.lens.cuda(), status=status,
                               out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert status.item() & kvq.DEV_BAD_PAGE
    assert torch.all(out[0, 1] == 0) and torch.any(out[0, 0] != 0)
    # a length beyond the page table
    status.zero_()
    out = kvq.decode_attention(p.shape, p.calib, p.cache, q, p.page_table.cuda(),
                               torch.tensor([40, 10 ** 6], dtype=torch.int32, device="cuda"), status=status)
    torch.cuda.synchronize()
    assert status.item() & kvq.DEV_BAD_LEN
    assert torch.all(out[0, 1] == 0)
    # a slot beyond the cache: skipped and flagged, the rest written
    status.zero_()
    before = p.cache.data.clone()
    k, v = synth.sequence_kv(w, 0, 0, 2, "cuda")
    slots = torch.tensor([p.num_pages * 16 + 3, 5], dtype=torch.int64, device="cuda")
    kvq.quantize_append(p.shape, p.calib, p.cache, k.contiguous(), v.contiguous(), slots, status=status)
    torch.cuda.synchronize()
    assert status.item() & kvq.DEV_BAD_SLOT
    changed = (p.cache.data != before).nonzero()
    assert changed.numel() > 0 and torch.all(changed[:, 1] == 0)           # only page 0 (slot 5) touched


def test_bad_page_in_a_split_unit(kvq):
    # A page id outside the pool in one split of a long sequence: the split
    # poisons its partial, the fused merge writes the row as zeros (not NaN)
    # and the status says why; the other sequence, also split, is unaffected.
    w = small(num_layers=1, batch=2, calib_windows=1, calib_len=64)
    lens = [3000, 2500]
    p = harness.build_problem(kvq, w, lens=lens)
    assert kvq.decode_workspace_bytes(p.shape, 1, 2, p.page_table.shape[1]) > 0     # split
    cal = harness.oracle_calibration(p)
    pt = p.page_table.clone()
    pt[0, 100] = p.num_pages + 7
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    q = synth.decode_queries(w, 0, 0)[None].cuda()
    out = kvq.decode_attention(p.shape, p.calib, p.cache, q, pt.cuda(), p.lens.cuda(), status=status,
                               out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert status.item() & kvq.DEV_BAD_PAGE
    assert torch.all(out[0, 0] == 0)
    want = harness.oracle_attend(p, 0, 1, q[0, 1].float().cpu().numpy()[None], lens[1] - 1, lens[1], cal)
    harness.check_attention(out[0, 1].cpu().numpy(), want[0], "split sequence beside a bad page f32")


def test_bounded_wait_gives_up_and_context_survives(kvq):
    """A wait on a barrier nothing arrives at runs out and reports DEV_TIMEOUT."""
    import time
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    kvq.selftest_wait_timeout(status, limit_ns=20_000_000)   # 20 ms
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert status.item() == kvq.DEV_TIMEOUT
    assert dt < 5.0
    # the context is still usable: a normal decode afterwards is correct
    w = small(num_layers=1, batch=1, calib_windows=1, calib_len=32)
    p = harness.build_problem(kvq, w, lens=[50])
    cal = harness.oracle_calibration(p)
    q, out = decode_all(kvq, p)
    want = harness.oracle_attend(p, 0, 0, q[0, 0][None], 49, 50, cal)
    harness.check_attention(out[0, 0], want[0], "decode after a timed-out wait f32")


@pytest.mark.parametrize("hkv,group,hadamard", [(1, 1, False), (2, 4, True), (4, 2, False), (8, 3, False),
                                                (6, 4, True)])
def test_other_head_shapes(kvq, hkv, group, hadamard):
    """kv heads 1..8 and GQA groups 1..4: append, decode and prefill."""
    w = small(num_layers=1, batch=2, calib_windows=1, calib_len=48, hadamard=hadamard,
              num_kv_heads=hkv, num_q_heads=hkv * group, prefill_chunk=40)
    lens = [70, 143]
    p = harness.build_problem(kvq, w, lens=lens)
    cal = harness.oracle_calibration(p)
    for got, want in zip(harness.calib_host(p), cal):
        np.testing.assert_array_equal(got, want)
    for b, n in enumerate(lens):
        assert_codes_equal(p, 0, b, n, cal)
    q, out = decode_all(kvq, p, out_dtype=torch.float32)
    for b, n in enumerate(lens):
        want = harness.oracle_attend(p, 0, b, q[0, b][None], n - 1, n, cal)
        harness.check_attention(out[0, b], want[0], f"decode hkv {hkv} g {group} seq {b} f32")
    qp = synth.prefill_queries(w, 0)[None]                       # [1][B][40][Hq][D]
    q_start = torch.tensor([n - 40 for n in lens], dtype=torch.int32)
    outp = kvq.prefill_attention(p.shape, p.calib, p.cache, qp.cuda(), q_start.cuda(), p.page_table.cuda(),
                                 p.lens.cuda(), out_dtype=torch.float32).cpu().numpy()
    for b, n in enumerate(lens):
        want = harness.oracle_attend(p, 0, b, qp[0, b].float().numpy(), n - 40, n, cal)
        harness.check_attention(outp[0, b], want, f"prefill hkv {hkv} g {group} seq {b} f32")
