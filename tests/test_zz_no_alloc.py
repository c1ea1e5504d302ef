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
    tag = "bf16" if out_dtype == torch.bfloat16 else "f32"
    for li in range(len(p.layers)):
        for b in range(len(p.lens)):
            harness.check_attention(out[li, b].float().cpu().numpy(), ref[li, b].float().cpu().numpy(),
                                    f"noalloc layer {li} seq {b} {tag}")


def test_noalloc_matches_workspace_decode_on_consecutive_calls(kvq):
    # first call: two layers, long ragged sequences, fp32 output
    p1 = _problem(kvq, [700, 1500, 33], layers=[0, 1])
    _compare(kvq, p1, step=0, out_dtype=torch.float32)
    # second call: a different, smaller problem that leaves the first call's
    # partials beyond its own in the array; bf16 output, rotated keys
    p2 = _problem(kvq, [400, 90], layers=[3], hadamard=True)
    _compare(kvq, p2, step=1, out_dtype=torch.bfloat16)


def test_noalloc_rejects_problems_beyond_the_scratch(kvq):
    import ctypes
    # few (layer, sequence) units over very long sequences: many splits
    shape = kvq.Shape(8, 32, 8)
    need = kvq.decode_workspace_bytes(shape, 8, 22, 16384)
    assert need > kvq.NOALLOC_SCRATCH_BYTES
    st = kvq._lib.kvq_decode_attention_noalloc(
        ctypes.byref(shape.c()), ctypes.byref(kvq._Calib(16, 16, 16, 16)),
        ctypes.byref(kvq._Cache(4096, 8 * 2304 * 4, 4)), 0, 8, 256, 1, 512, 16384, 768, 22, 1024, 1, None, None)
    assert st == kvq.KVQ_EWORKSPACE
