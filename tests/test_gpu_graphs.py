"""The hot path under CUDA-graph capture and on concurrent streams.

A serving loop captures a decode step once and replays it with new inputs
copied into the captured buffers.  Every call of the library is stream-ordered
and allocates nothing when its buffers are given, so one step -- append one
token per sequence into every layer, then decode every layer (split-K with
the combine on this small batch) -- and a chunked prefill (fp16 and FP4 Q.K)
are captured with torch.cuda.CUDAGraph and replayed.  Each replay must equal
the eager call on a copy of the cache bit for bit: the same kernels in the
same launch shapes, deterministic reductions.  Two problems run at once on two
streams give their sequential results bit for bit (the library keeps no state).
"""
import dataclasses

import pytest
import torch

import harness
import synth

pytestmark = pytest.mark.gpu


def _small(**kw):
    return dataclasses.replace(synth.WORKLOADS["qwen3_8b"], **kw)


def _capture(fn):
    g = torch.cuda.CUDAGraph()
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        fn()
    return g


def test_decode_step_graph_replay_matches_eager(kvq):
    w = _small(num_layers=2, batch=3, calib_windows=1, calib_len=64)
    lens = torch.tensor([40, 77, 130], dtype=torch.int32)
    steps = 3
    p = harness.build_problem(kvq, w, lens=lens, extra_tokens=steps, keep_tails=True)
    tk, tv = p.tails                                           # [steps][nl][B][Hkv][D]
    nl, B = 2, 3
    pt = p.page_table.cuda()
    eager_cache = kvq.PagedCache(p.cache.data.clone())
    qs = [torch.stack([synth.decode_queries(w, l, e, "cuda") for l in range(nl)]) for e in range(steps)]

    def slots_for(e):
        return torch.cat([synth.slot_mapping(p.page_table, torch.tensor([b]), torch.tensor([int(lens[b]) + e]))
                          for b in range(B)]).cuda()

    # eager reference on the copy
    want = []
    for e in range(steps):
        kvq.quantize_append(p.shape, p.calib, eager_cache, tk[e].contiguous(), tv[e].contiguous(), slots_for(e))
        want.append(kvq.decode_attention(p.shape, p.calib, eager_cache, qs[e], pt, (lens + e + 1).cuda(),
                                         out_dtype=torch.float32).clone())
    # the captured step on the original cache
    k_buf, v_buf = torch.empty_like(tk[0]), torch.empty_like(tv[0])
    slot_buf = torch.empty(B, dtype=torch.int64, device="cuda")
    q_buf = torch.empty_like(qs[0])
    len_buf = torch.empty(B, dtype=torch.int32, device="cuda")
    out_buf = torch.empty(q_buf.shape, dtype=torch.float32, device="cuda")
    ws = kvq.new_workspace(kvq.decode_workspace_bytes(p.shape, nl, B, pt.shape[1]))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")

    def step():
        kvq.quantize_append(p.shape, p.calib, p.cache, k_buf, v_buf, slot_buf, status=status)
        kvq.decode_attention(p.shape, p.calib, p.cache, q_buf, pt, len_buf, out=out_buf, workspace=ws,
                             status=status)

    g = _capture(step)
    for e in range(steps):
        k_buf.copy_(tk[e])
        v_buf.copy_(tv[e])
        slot_buf.copy_(slots_for(e))
        q_buf.copy_(qs[e])
        len_buf.copy_(lens + e + 1)
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out_buf, want[e]), f"step {e}"
    assert status.item() == 0
    assert torch.equal(p.cache.data, eager_cache.data)


@pytest.mark.parametrize("fp4", [False, True])
def test_prefill_graph_replay_matches_eager(kvq, fp4):
    w = _small(num_layers=2, batch=2, calib_windows=1, calib_len=64, prefill_chunk=48)
    P0, Tq = [100, 33], 48
    lens = torch.tensor([n + Tq for n in P0], dtype=torch.int32)
    p = harness.build_problem(kvq, w, lens=lens)
    pt, ln = p.page_table.cuda(), lens.cuda()
    q_start = torch.tensor(P0, dtype=torch.int32, device="cuda")
    q_buf = torch.empty(2, 2, Tq, w.num_q_heads, w.head_dim, dtype=torch.bfloat16, device="cuda")
    out_buf = torch.empty(q_buf.shape, dtype=torch.float32, device="cuda")

    def run(q, out=None):
        return kvq.prefill_attention(p.shape, p.calib, p.cache, q, q_start, pt, ln, out=out,
                                     out_dtype=torch.float32, qk_fp4=fp4)

    g = _capture(lambda: run(q_buf, out_buf))
    for seed_layer in (0, 1):
        q = torch.stack([synth.prefill_queries(w, (l + seed_layer) % 2, "cuda") for l in range(2)])
        want = run(q).clone()
        q_buf.copy_(q)
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out_buf, want)


def test_concurrent_streams_match_sequential(kvq):
    # the library keeps no state: two problems decoded (and prefilled) at the
    # same time on two streams give the sequential results bit for bit
    w = _small(num_layers=2, batch=3, calib_windows=1, calib_len=64, prefill_chunk=32)
    probs = [harness.build_problem(kvq, w, lens=[40 + 30 * i, 90, 200 - 50 * i]) for i in range(2)]
    qd = torch.stack([synth.decode_queries(w, l, 0, "cuda") for l in range(2)])
    qp = torch.stack([synth.prefill_queries(w, l, "cuda") for l in range(2)])

    def run(p):
        ln = p.lens.cuda()
        d = kvq.decode_attention(p.shape, p.calib, p.cache, qd, p.page_table.cuda(), ln, out_dtype=torch.float32)
        qs = (ln - 32).clamp_min(0).to(torch.int32)
        f = kvq.prefill_attention(p.shape, p.calib, p.cache, qp, qs, p.page_table.cuda(), ln,
                                  out_dtype=torch.float32)
        return d, f

    want = [run(p) for p in probs]
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream() for _ in probs]
    got = []
    for p, s in zip(probs, streams):
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            got.append(run(p))
    torch.cuda.synchronize()
    for (d0, f0), (d1, f1) in zip(want, got):
        assert torch.equal(d0, d1) and torch.equal(f0, f1)


def test_noalloc_decode_graph_replay(kvq):
    # the allocation-free entry point under capture: its first call (which
    # looks up the static scratch array) is made before the capture
    w = _small(num_layers=2, batch=3, calib_windows=1, calib_len=64)
    lens = torch.tensor([40, 77, 130], dtype=torch.int32)
    p = harness.build_problem(kvq, w, lens=lens)
    pt, ln = p.page_table.cuda(), lens.cuda()
    q_buf = torch.stack([synth.decode_queries(w, l, 0, "cuda") for l in range(2)])
    out_buf = torch.empty(q_buf.shape, dtype=torch.float32, device="cuda")
    kvq.decode_attention_noalloc(p.shape, p.calib, p.cache, q_buf, pt, ln, out_buf)   # before capture
    g = _capture(lambda: kvq.decode_attention_noalloc(p.shape, p.calib, p.cache, q_buf, pt, ln, out_buf))
    for step in (1, 2):
        q = torch.stack([synth.decode_queries(w, l, step, "cuda") for l in range(2)])
        want = kvq.decode_attention(p.shape, p.calib, p.cache, q, pt, ln, out_dtype=torch.float32)
        q_buf.copy_(q)
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out_buf, want)
