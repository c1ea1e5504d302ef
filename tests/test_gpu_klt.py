"""Static per-head KLT on the GPU against the oracle ("NVFP4 attention cache
on W4A4 Qwen3-8B", results table rows "K: static per-head KLT" and "K:
static KLT + smoothing").

Two kinds of check:
  - kvq_calibrate_klt as a calibration.  Its basis comes out of an fp32
    Jacobi eigensolver on the device, the oracle's out of fp64 eigh; the two
    are compared as bases (orthogonal, diagonalising the second moment, same
    order and signs, each vector close to the oracle's where the eigenvalue
    gap makes it well defined).  The smoothing factors are compared bit for
    bit, and the tensor scales bit for bit given the basis the device chose
    (an eigenbasis is not unique where eigenvalues nearly coincide).
  - The append, decode and both prefills on the ORACLE's calibration: its
    eigh basis rounded to fp32, its smoothing and its tensor scales are
    written into a caller-owned Calibration (tests/harness.py), so the oracle
    side of every comparison reads no value computed on the device.  Codes
    and scales bit for bit, attention within the stated tolerance.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu


def _windows(layers=2, windows=4, length=128):
    w = dataclasses.replace(synth.WORKLOADS["qwen3_8b"], num_layers=layers, calib_windows=windows,
                            calib_len=length)
    win = [synth.calibration_windows(w, l) for l in range(layers)]
    return w, torch.stack([x[0] for x in win]), torch.stack([x[1] for x in win])


@pytest.mark.parametrize("exclude_pos0", [True, False])
def test_klt_calibration_matches_oracle(kvq, exclude_pos0):
    # exclude_pos0 False: "K: same smoothing, but sink token included in the
    # absmax" (results table), here for the smoothing and the second moment
    w, kc, vc = _windows()
    shape = kvq.Shape(2, w.num_q_heads, w.num_kv_heads, use_klt=True)
    cal = kvq.calibrate_klt(shape, kc.cuda().contiguous(), vc.cuda().contiguous(), exclude_pos0=exclude_pos0)
    torch.cuda.synchronize()
    k, v = kc.float().numpy(), vc.float().numpy()
    s_o, inv_o, U_o, ev_o = oracle.calibrate_klt(k, v, exclude_pos0=exclude_pos0)
    np.testing.assert_array_equal(cal.k_smooth.cpu().numpy(), s_o)
    np.testing.assert_array_equal(cal.k_inv_smooth.cpu().numpy(), inv_o)
    U = cal.k_klt.cpu().numpy()
    t0 = 1 if exclude_pos0 else 0
    for l in range(2):
        y = oracle.transform_keys(k[l, :, t0:].reshape(-1, 8, 128), inv_o[l])
        for h in range(8):
            u = U[l, h].astype(np.float64)
            np.testing.assert_allclose(u.T @ u, np.eye(128), atol=2e-5)
            C = y[:, h].astype(np.float64).T @ y[:, h].astype(np.float64)
            D = u.T @ C @ u
            lam = np.diag(D)
            assert np.abs(D - np.diag(lam)).max() <= 2e-5 * lam.max(), (l, h)
            assert np.all(np.diff(lam) <= 1e-5 * lam.max()), (l, h)        # decreasing
            assert np.all(u[np.argmax(np.abs(u), axis=0), np.arange(128)] > 0)
            # vector by vector against fp64 eigh where the relative gap is wide
            lo = ev_o[l, h] * y.shape[0]                                 # oracle's C is / N
            gap = np.minimum(np.abs(np.diff(lo, prepend=np.inf)), np.abs(np.diff(lo, append=-np.inf)))
            wide = gap > 1e-3 * lo.max()
            dots = np.abs(np.sum(u * U_o[l, h].astype(np.float64), axis=0))
            assert np.all(dots[wide] > 1 - 1e-4), (l, h, dots[wide].min())
    # the value scale does not depend on the basis: bit for bit; the key
    # scale is a function of the basis the device chose: bit for bit given
    # it, and within the basis' own tolerance of the oracle's eigh basis
    gk, gv = oracle.klt_tensor_scales(k, v, inv_o, U)
    np.testing.assert_array_equal(cal.k_gscale.cpu().numpy(), gk)
    np.testing.assert_array_equal(cal.v_gscale.cpu().numpy(), gv)
    gk_o, gv_o = oracle.klt_tensor_scales(k, v, inv_o, U_o)
    np.testing.assert_array_equal(gv, gv_o)
    np.testing.assert_allclose(gk, gk_o, rtol=1e-3)


def _klt_problem(kvq, lens, layers=2, exclude_pos0=True):
    import harness
    w = dataclasses.replace(synth.WORKLOADS["qwen3_8b"], num_layers=layers, batch=len(lens), calib_windows=4,
                            calib_len=128)
    return harness.build_problem(kvq, w, lens=lens, klt=True, exclude_pos0=exclude_pos0)


@pytest.mark.parametrize("exclude_pos0", [True, False])
def test_klt_append_codes_bit_exact(kvq, exclude_pos0):
    import harness
    lens = [5, 150, 301]
    p = _klt_problem(kvq, lens, exclude_pos0=exclude_pos0)
    cal = harness.checked_calibration(p)
    for li in range(2):
        layer = p.cache.data[li].cpu().numpy()
        for b, n in enumerate(lens):
            got = harness.read_tokens(layer, 8, p.page_table[b].numpy(), n)
            want = harness.oracle_sequence(p, li, b, n, cal)
            for name, g in zip(("kc", "ksf", "vc", "vsf"), got):
                np.testing.assert_array_equal(g, want[name], err_msg=f"{name} layer {li} seq {b}")


def test_klt_decode_within_tolerance(kvq):
    import harness
    lens = [5, 150, 301]
    p = _klt_problem(kvq, lens)
    cal = harness.checked_calibration(p)
    q = torch.stack([synth.decode_queries(p.w, l, 0) for l in p.layers])
    for dt, tag in ((torch.float32, "f32"), (torch.bfloat16, "bf16")):
        out = kvq.decode_attention(p.shape, p.calib, p.cache, q.cuda(), p.page_table.cuda(), p.lens.cuda(),
                                   out_dtype=dt).float().cpu().numpy()
        for li in range(2):
            for b, n in enumerate(lens):
                want = harness.oracle_attend(p, li, b, q[li, b].float().numpy()[None], n - 1, n, cal)
                harness.check_attention(out[li, b], want[0], f"klt decode layer {li} seq {b} {tag}")


@pytest.mark.parametrize("qk_fp4", [False, True])
def test_klt_prefill_within_tolerance(kvq, qk_fp4):
    import harness
    w = dataclasses.replace(synth.WORKLOADS["qwen3_8b"], num_layers=2, batch=2, calib_windows=4, calib_len=128,
                            prefill_chunk=48)
    P0, Tq = [100, 33], 48
    lens = [n + Tq for n in P0]
    p = harness.build_problem(kvq, w, lens=lens, klt=True)
    cal = harness.checked_calibration(p)
    q = torch.stack([synth.prefill_queries(w, l) for l in p.layers])
    q_start = torch.tensor(P0, dtype=torch.int32)
    out = kvq.prefill_attention(p.shape, p.calib, p.cache, q.cuda(), q_start.cuda(), p.page_table.cuda(),
                                p.lens.cuda(), out_dtype=torch.float32, qk_fp4=qk_fp4).float().cpu().numpy()
    attend = harness.oracle_attend_fp4q if qk_fp4 else harness.oracle_attend
    for li in range(2):
        for b in range(2):
            want = attend(p, li, b, q[li, b].float().numpy(), P0[b], lens[b], cal)
            harness.check_attention(out[li, b], want, f"klt prefill{' fp4' if qk_fp4 else ''} layer {li} seq {b}")


def test_klt_append_bad_slot_skipped_and_flagged(kvq):
    """A slot beyond the cache in a KLT append: the key kernel (and the value
    kernel) skip it and set KVQ_DEV_BAD_SLOT; the other token is written."""
    p = _klt_problem(kvq, [40])
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    before = p.cache.data.clone()
    k, v = synth.sequence_kv(p.w, 0, 0, 2, "cuda")
    slots = torch.tensor([p.num_pages * 16 + 3, 5], dtype=torch.int64, device="cuda")
    kvq.quantize_append(p.shape, p.calib, p.cache, k.contiguous(), v.contiguous(), slots, status=status)
    torch.cuda.synchronize()
    assert status.item() & kvq.DEV_BAD_SLOT
    changed = (p.cache.data != before).nonzero()
    # only layer 0's page 0 (slot 5) is touched
    assert changed.numel() > 0 and torch.all(changed[:, 0] == 0) and torch.all(changed[:, 1] == 0)
