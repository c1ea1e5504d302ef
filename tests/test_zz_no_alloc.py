"""kvq_decode_attention_noalloc against kvq_decode_attention.

The allocation-free entry point serves callers that cannot allocate device
memory (a host runtime that owns the device-memory budget, or a path that
cannot afford cudaMalloc's implicit synchronisation): its split-K scratch is
a static device array inside the library.  It must give the same results as
the regular entry point given a caller-allocated workspace, also on a second
call that finds the previous call's partials still in the array.

This file is named to be collected last, and passes both alone in a fresh
process and after the rest of the suite.
"""
import dataclasses

import pytest
import torch

import harness
import synth

pytestmark = pytest.mark.gpu


def _problem(kvq, lens, layers, name="qwen3_8b", hadamard=False):
    w = dataclasses.replace(synth.WORKLOADS[name], num_layers=max(layers) + 1, batch=len(lens),
                            calib_windows=1, calib_len=64, hadamard=hadamard)
    return harness.build_problem(kvq, w, lens=lens, layers=layers, keep_host=False)


def _compare(kvq, p, step, out_dtype):
    q = torch.stack([synth.decode_queries(p.w, l, step) for l in p.layers]).cuda()
    pt, lens = p.page_table.cuda(), p.lens.cuda()
    need = kvq.decode_workspace_bytes(p.shape, len(p.layers), len(p.lens), pt.shape[1])
    assert 0 < need <= kvq.NOALLOC_SCRATCH_BYTES           # the split-K scratch is in use
    ref = kvq.decode_attention(p.shape, p.calib, p.cache, q, pt, lens, out_dtype=out_dtype)
    out = torch.full_like(ref, float("nan"))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    kvq.decode_attention_noalloc(p.shape, p.calib, p.cache, q, pt, lens, out, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    # the same kernels with the same split plan, only the scratch differs:
    # the results are identical
    assert torch.equal(out, ref), (out - ref).abs().max().item()


def test_noalloc_matches_workspace_decode_on_consecutive_calls(kvq):
    # first call: two layers, long ragged sequences, fp32 output
    p1 = _problem(kvq, [700, 1500, 33], layers=[0, 1])
    _compare(kvq, p1, step=0, out_dtype=torch.float32)
    # second call: a different, smaller problem that leaves the first call's
    # partials beyond its own in the array; bf16 output, rotated keys
    p2 = _problem(kvq, [400, 90], layers=[3], hadamard=True)
    _compare(kvq, p2, step=1, out_dtype=torch.bfloat16)


def test_noalloc_rejects_problems_beyond_the_scratch(kvq):
    # few (layer, sequence) units over very long page tables: many splits,
    # more partials than the static array holds.  Every buffer is real and
    # sized for the problem (a 4-page cache, sequences of one token), so
    # even a launch would stay in bounds; the call must refuse it.
    L, B, maxp = 8, 22, 16384
    shape = kvq.Shape(L, 32, 8)
    need = kvq.decode_workspace_bytes(shape, L, B, maxp)
    assert need > kvq.NOALLOC_SCRATCH_BYTES
    calib = kvq.new_calibration(shape)
    calib.k_smooth.fill_(1.0)
    calib.k_inv_smooth.fill_(1.0)
    calib.k_gscale.fill_(1.0)
    calib.v_gscale.fill_(1.0)
    cache = kvq.new_cache(shape, 4)
    cache.data.zero_()
    q = torch.zeros(L, B, 32, 128, dtype=torch.float32, device="cuda")
    pt = torch.zeros(B, maxp, dtype=torch.int32, device="cuda")
    lens = torch.ones(B, dtype=torch.int32, device="cuda")
    out = torch.full((L, B, 32, 128), 7.0, dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(kvq.KVQError) as e:
        kvq.decode_attention_noalloc(shape, calib, cache, q, pt, lens, out, status=status)
    assert e.value.status == kvq.KVQ_EWORKSPACE
    torch.cuda.synchronize()
    assert status.item() == 0 and torch.all(out == 7.0)     # nothing was launched
