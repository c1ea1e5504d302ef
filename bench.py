#!/usr/bin/env python
"""Throughput of the NVFP4 attention-cache hot path on B200; prints one JSON line.

Default workload (N=1): ragged decode -- 36 layers, 32 query / 8 KV heads,
head_dim 128, batch 64 with lengths uniform on [1024, 8192], a paged NVFP4
cache of 16-token pages in shuffled order.  One step = append one new token
per sequence into every layer (kvq_quantize_append) + one decode of every
layer (kvq_decode_attention).  The 64 steps of the workload are cycled.
After the headline, the line's "secondary" entry carries the kernel numbers
of the other workloads (chunked prefill with fp16 and FP4 Q.K, the qwen3_8b
and hadamard prefix workloads), each measured with a few steps in the same
run.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kvq|reference]

With N > 1 (torchrun) every rank runs its own replica of the workload (the
path has no exchange step: independent sequences); the reported value is the
sum over ranks, timed as the max over ranks.  ``--impl reference`` times the
CPU oracle on bounded samples of the same workload instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = "NVFP4-KV decode attention tokens/s; achieved HBM GB/s vs B200 peak"
FALLBACK_HBM_GBS = 6650.0
TOKEN_LAYER_BYTES = 1152          # packed K+V codes and scales of 8 heads
TOKEN_LAYER_BYTES_BF16K = 2624    # mixed cache: bf16 keys (8 x 256 B) + packed values (8 x 72 B)
QO_BYTES_PER_SEQ_LAYER = 32 * 128 * 2 * 2   # bf16 query in + bf16 output
# what the kernels compute in ("dtype" of the JSON line)
DECODE_DTYPE = ("fp16 mma operands (exact e2m1 x e4m3 dequant, query split hi + lo, P rounded to fp16), "
                "f32 accumulate")
PREFILL_DTYPE_F16 = "fp16 tcgen05 operands (exact dequant, query split hi + lo, P fp16), f32 accumulate"
PREFILL_DTYPE_FP4 = "nvfp4 Q.K (query quantised per row) + fp16 P.V, f32 accumulate"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="kvq", choices=["kvq", "reference"])
    ap.add_argument("--workload", default="ragged", choices=["ragged", "prefill", "qwen3_8b", "hadamard"],
                    help="ragged (default, the decode-throughput workload); prefill, qwen3_8b, hadamard: "
                         "the chunked-prefill and prefix workloads, for their own kernel numbers")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--klt", action="store_true",
                    help="ragged workload with smoothing plus the static per-head KLT of the keys")
    ap.add_argument("--k-format", default="nvfp4", choices=["nvfp4", "bf16"],
                    help="key storage of the ragged workload: packed NVFP4, or bf16 keys with NVFP4 values")
    ap.add_argument("--qk", default="fp16", choices=["fp16", "fp4"],
                    help="Q.K of the prefill workload: fp16 (query hi + lo) or block-scaled FP4 (query quantised)")
    ap.add_argument("--source-sha", action="store_true",
                    help="print the hash of the decode kernel's sources (the key of the committed ncu counters) and exit")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the other workloads' kernel numbers (prefill fp16 / FP4 Q.K, qwen3_8b, hadamard) "
                         "measured after the headline")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--layers", type=int, default=36,
                    help="layers of the ragged workload (36; fewer only for profiling captures)")
    return ap.parse_args()


# ------------------------------------------------------------------ distributed
def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """SM clock and clock-event reasons of this process's GPU, sampled every
    5 ms from a background thread through NVML (reads only) while the timed
    region runs; nvidia-smi's own sampling loop where NVML is unavailable.
    The device is found by its UUID, so a remapped CUDA_VISIBLE_DEVICES cannot
    point the sampler at another GPU."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index: int):
        import threading
        self.proc = None
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            h = pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            self._nvml, self._h = pynvml, h
            self._thread = threading.Thread(target=self._poll, daemon=True)
            self._thread.start()
            return
        except Exception:
            self._thread = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", str(device_index)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def _sample(self) -> bool:
        nv, h = self._nvml, self._h
        try:
            self.samples.append((float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)),
                                 int(nv.nvmlDeviceGetCurrentClocksEventReasons(h))))
            return True
        except Exception:
            return False

    def _poll(self):
        # every 5 ms while the timed region runs (the thread may be scheduled
        # late while the main thread holds the interpreter; stop() adds a
        # closing sample, so a short region still has its two ends)
        while not self._stop.is_set():
            if not self._sample():
                return
            self._stop.wait(0.005)

    def stop(self):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=5)
            self._sample()
            if not self.samples:
                return None
            reasons = sorted({name for _, bits in self.samples for bit, name in self.REASONS.items() if bits & bit})
            return {"sm_mhz": statistics.median(m for m, _ in self.samples), "sm_max_mhz": self.max_mhz,
                    "reasons": reasons, "samples": len(self.samples), "source": "nvml, 5 ms"}
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [r.split(", ") for r in out.strip().splitlines() if r.count(",") >= 8]
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.strip() == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows), "source": "nvidia-smi, 200 ms"}


def measured_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


# every source of the decode kernel's translation unit: a change to any of
# them invalidates the committed ncu counters
DECODE_SOURCES = ("kvq_decode_tc.cu", "kvq_decode.cu", "kvq_attn.cuh", "kvq_common.cuh", "kvq_sync.cuh")


def decode_source_sha() -> str:
    h = hashlib.sha256()
    for name in DECODE_SOURCES:
        with open(os.path.join(ROOT, "bit_attention_decode_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic():
    """Per-launch DRAM bytes of the decode kernel from the committed ncu
    counters (profiles/decode_ragged_ncu.json), or None when the kernel's
    sources changed since that capture."""
    path = os.path.join(ROOT, "profiles", "decode_ragged_ncu.json")
    try:
        with open(path) as f:
            vals = json.load(f)
        if vals.get("kernel_source_sha256_16") != decode_source_sha():
            return None
        return float(vals["dram_bytes_per_full_launch"])
    except (OSError, KeyError, ValueError):
        return None


def fp32_fma_peak_tflops():
    """FP32 FMA peak from unit counts and clocks: 128 FMA lanes per SM per
    clock x SMs x the maximum SM clock (148 x 128 x 1.965 GHz = 37.2 TFMA/s
    on B200)."""
    try:
        import pynvml
        pynvml.nvmlInit()
        h = pynvml.nvmlDeviceGetHandleByIndex(torch.cuda.current_device())
        mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
    except Exception:
        mhz = 1965
    sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    return sms * 128 * mhz * 1e6 / 1e12


def append_entry(wl, peak_hbm):
    """The bulk append's line: HBM-bound, except with the KLT, whose key
    transform (16,384 FMAs per token-head) makes it bound by the FP32 FMA pipe."""
    ms = statistics.median(wl.append_ms)
    gbs = wl.append_bytes / (ms / 1e3) / 1e9
    d = {"kernel": "kvq quantize-append (bulk prefix, one layer per launch)", "alg_bytes_per_launch": wl.append_bytes,
         "achieved": gbs, "unit": "GB/s", "frac": gbs / peak_hbm, "bound": "hbm"}
    if wl.klt:
        fma = wl.prefix_tokens * wl.w.num_kv_heads * 128 * 128      # the key transform, per launch
        tfma = fma / (ms / 1e3) / 1e12
        pk = fp32_fma_peak_tflops()
        d.update({"bound": "alu", "alu_achieved": tfma, "alu_peak": pk, "alu_unit": "TFMA/s", "alu_frac": tfma / pk,
                  "alu_peak_source": "derived: SMs x 128 FP32 FMA lanes x max SM clock",
                  "alg_fma_per_launch": fma})
    return d


# ------------------------------------------------------------------ workload
class Ragged:
    """Device-resident ragged decode workload (one replica)."""

    def __init__(self, kvq, synth, layers=36, k_format=0, klt=False):
        self.kvq = kvq
        import dataclasses
        w = dataclasses.replace(synth.WORKLOADS["ragged"], num_layers=layers)
        self.k_format = k_format
        self.klt = klt
        self.tlb = TOKEN_LAYER_BYTES_BF16K if k_format else TOKEN_LAYER_BYTES
        self.w = w
        L, B, S = w.num_layers, w.batch, w.decode_steps
        self.L, self.B, self.S = L, B, S
        dev = "cuda"
        self.lens = synth.ragged_lengths(w)                          # [B] int32
        cap = self.lens + S
        self.page_table, self.num_pages = synth.build_page_table(w, cap)
        self.shape = kvq.Shape(L, w.num_q_heads, w.num_kv_heads, k_format=k_format, use_klt=klt)
        kc = torch.stack([synth.calibration_windows(w, l, dev)[0] for l in range(L)])
        vc = torch.stack([synth.calibration_windows(w, l, dev)[1] for l in range(L)])
        if klt:
            self.calib = kvq.calibrate_klt(self.shape, kc, vc, exclude_pos0=True)
        else:
            self.calib = kvq.calibrate_smoothing(self.shape, kc, vc, exclude_pos0=True)
        del kc, vc
        self.cache = kvq.new_cache(self.shape, self.num_pages, dev)
        H, D = w.num_kv_heads, w.head_dim
        self.k_new = torch.empty(S, L, B, H, D, dtype=torch.bfloat16, device=dev)
        self.v_new = torch.empty_like(self.k_new)
        pos = torch.arange(S)[:, None] + self.lens[None, :].long()          # [S][B]
        seq = torch.arange(B)[None, :].expand(S, B)
        self.slots = synth.slot_mapping(self.page_table, seq.reshape(-1), pos.reshape(-1)).view(S, B).to(dev)
        prefix_slots = torch.cat([synth.slot_mapping(self.page_table, torch.full((int(n),), b), torch.arange(int(n)))
                                  for b, n in enumerate(self.lens.tolist())]).to(dev)
        self.prefix_tokens = int(self.lens.sum())
        for l in range(L):
            ks, vs = [], []
            for b, n in enumerate(self.lens.tolist()):
                k, v = synth.sequence_kv(w, l, b, n + S, dev)
                ks.append(k[:n])
                vs.append(v[:n])
                self.k_new[:, l, b] = k[n:]
                self.v_new[:, l, b] = v[n:]
            kc_all, vc_all = torch.cat(ks), torch.cat(vs)
            kvq.quantize_append(self.shape, self.calib, self.cache, kc_all, vc_all, prefix_slots, layer0=l)
            del ks, vs
            if l == L - 1:
                # the last layer's prefix, kept to time the bulk append (time_bulk_append)
                self.bulk = (kc_all, vc_all, prefix_slots, l)
            del kc_all, vc_all
        self.q = torch.stack([torch.stack([synth.decode_queries(w, l, s, dev) for l in range(L)])
                              for s in range(S)])                             # [S][L][B][Hq][D]
        self.seq_lens = (self.lens[None, :] + torch.arange(1, S + 1)[:, None]).to(torch.int32).to(dev)
        self.page_table_dev = self.page_table.to(dev)
        self.out = torch.empty(L, B, w.num_q_heads, D, dtype=torch.bfloat16, device=dev)
        need = kvq.decode_workspace_bytes(self.shape, L, B, self.page_table.shape[1])
        self.ws = kvq.new_workspace(need, dev)
        # append (+ KLT keys) and decode (+ KLT queries); a split decode merges in the same launch
        self.launches_per_step = 4 if klt else 2
        torch.cuda.synchronize()
        # bulk append of each layer's prefix (read bf16 K and V, write codes + scales)
        self.append_bytes = self.prefix_tokens * (2 * w.num_kv_heads * D * 2 + self.tlb)

    def time_bulk_append(self, reps: int = 6):
        """CUDA-event times of the bulk prefix append of one layer (1.54 GB moved
        at 36 layers x 64 sequences): re-appending the same tokens rewrites
        identical bytes; launches go back to back so the queue never drains."""
        kc_all, vc_all, slots, l = self.bulk
        torch.cuda.synchronize()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(reps + 1)]
        ev[0].record()
        for r in range(reps):
            self.kvq.quantize_append(self.shape, self.calib, self.cache, kc_all, vc_all, slots, layer0=l)
            ev[r + 1].record()
        torch.cuda.synchronize()
        # the first launch is a warm-up
        self.append_ms = [ev[r].elapsed_time(ev[r + 1]) for r in range(1, reps)]

    def decode_bytes(self, s: int) -> int:
        valid = int(self.lens.sum()) + self.B * (s + 1)
        return valid * self.L * self.tlb + self.B * self.L * QO_BYTES_PER_SEQ_LAYER

    def append(self, s: int):
        self.kvq.quantize_append(self.shape, self.calib, self.cache, self.k_new[s], self.v_new[s], self.slots[s])

    def decode(self, s: int):
        self.kvq.decode_attention(self.shape, self.calib, self.cache, self.q[s], self.page_table_dev,
                                  self.seq_lens[s], out=self.out, workspace=self.ws)


class Prefill:
    """Chunked causal prefill: 36 layers, batch 8, 8192 cached tokens + a
    512-token chunk.  One step = append the chunk's K/V into every layer, then
    prefill attention of every layer (tcgen05)."""

    def __init__(self, kvq, synth, layers=36, k_format=0, qk_fp4=False):
        import dataclasses
        w = dataclasses.replace(synth.WORKLOADS["prefill"], num_layers=layers)
        self.k_format = k_format
        self.qk_fp4 = qk_fp4
        self.kvq, self.w = kvq, w
        L, B, P0, Tq = w.num_layers, w.batch, w.context, w.prefill_chunk
        self.L, self.B, self.P0, self.Tq = L, B, P0, Tq
        dev = "cuda"
        total = P0 + Tq
        lens = torch.full((B,), total, dtype=torch.int32)
        self.page_table, self.num_pages = synth.build_page_table(w, lens)
        self.shape = kvq.Shape(L, w.num_q_heads, w.num_kv_heads, k_format=k_format)
        kc = torch.stack([synth.calibration_windows(w, l, dev)[0] for l in range(L)])
        vc = torch.stack([synth.calibration_windows(w, l, dev)[1] for l in range(L)])
        self.calib = kvq.calibrate_smoothing(self.shape, kc, vc, exclude_pos0=True)
        del kc, vc
        self.cache = kvq.new_cache(self.shape, self.num_pages, dev)
        H, D = w.num_kv_heads, w.head_dim
        pre_slots = torch.cat([synth.slot_mapping(self.page_table, torch.full((P0,), b), torch.arange(P0))
                               for b in range(B)]).to(dev)
        self.chunk_slots = torch.cat([synth.slot_mapping(self.page_table, torch.full((Tq,), b),
                                                         torch.arange(P0, total)) for b in range(B)]).to(dev)
        self.chunk_k = torch.empty(L, B * Tq, H, D, dtype=torch.bfloat16, device=dev)
        self.chunk_v = torch.empty_like(self.chunk_k)
        for l in range(L):
            ks, vs = [], []
            for b in range(B):
                k, v = synth.sequence_kv(w, l, b, total, dev)
                ks.append(k[:P0])
                vs.append(v[:P0])
                self.chunk_k[l, b * Tq:(b + 1) * Tq] = k[P0:]
                self.chunk_v[l, b * Tq:(b + 1) * Tq] = v[P0:]
            kvq.quantize_append(self.shape, self.calib, self.cache, torch.cat(ks), torch.cat(vs), pre_slots, layer0=l)
            del ks, vs
        self.q = torch.stack([synth.prefill_queries(w, l, dev) for l in range(L)])   # [L][B][Tq][Hq][D]
        self.q_start = torch.full((B,), P0, dtype=torch.int32, device=dev)
        self.seq_lens = lens.to(dev)
        self.pt = self.page_table.to(dev)
        self.out = torch.empty_like(self.q)
        # attended keys summed over the chunk's queries, per (layer, sequence, query head)
        keys = Tq * P0 + Tq * (Tq + 1) // 2
        self.flops = 4 * D * w.num_q_heads * L * B * keys
        torch.cuda.synchronize()

    def append(self):
        self.kvq.quantize_append(self.shape, self.calib, self.cache, self.chunk_k, self.chunk_v, self.chunk_slots)

    def attend(self):
        self.kvq.prefill_attention(self.shape, self.calib, self.cache, self.q, self.q_start, self.pt, self.seq_lens,
                                   out=self.out, qk_fp4=self.qk_fp4)


class Prefix:
    """Qwen3-8B-shaped (or Hadamard) prefix workload: one step = quantise-append
    every layer's whole prefix (one launch), then one decode step of every layer."""

    def __init__(self, kvq, synth, name, layers=36):
        import dataclasses
        w = dataclasses.replace(synth.WORKLOADS[name], num_layers=layers)
        self.kvq, self.w = kvq, w
        L, B, T = w.num_layers, w.batch, w.context
        self.L, self.B, self.T = L, B, T
        dev = "cuda"
        lens = torch.full((B,), T, dtype=torch.int32)
        self.page_table, self.num_pages = synth.build_page_table(w, lens)
        self.shape = kvq.Shape(L, w.num_q_heads, w.num_kv_heads, use_hadamard=w.hadamard)
        kc = torch.stack([synth.calibration_windows(w, l, dev)[0] for l in range(L)])
        vc = torch.stack([synth.calibration_windows(w, l, dev)[1] for l in range(L)])
        self.calib = kvq.calibrate_smoothing(self.shape, kc, vc, exclude_pos0=True)
        del kc, vc
        self.cache = kvq.new_cache(self.shape, self.num_pages, dev)
        H, D = w.num_kv_heads, w.head_dim
        self.slots = torch.cat([synth.slot_mapping(self.page_table, torch.full((T,), b), torch.arange(T))
                                for b in range(B)]).to(dev)
        self.k = torch.empty(L, B * T, H, D, dtype=torch.bfloat16, device=dev)
        self.v = torch.empty_like(self.k)
        for l in range(L):
            for b in range(B):
                k, v = synth.sequence_kv(w, l, b, T, dev)
                self.k[l, b * T:(b + 1) * T] = k
                self.v[l, b * T:(b + 1) * T] = v
        self.q = torch.stack([synth.decode_queries(w, l, 0, dev) for l in range(L)])
        self.seq_lens = lens.to(dev)
        self.pt = self.page_table.to(dev)
        self.out = torch.empty(L, B, w.num_q_heads, D, dtype=torch.bfloat16, device=dev)
        need = kvq.decode_workspace_bytes(self.shape, L, B, self.page_table.shape[1])
        self.ws = kvq.new_workspace(need, dev)
        self.launches = 2
        self.append_bytes = L * B * T * (2 * H * D * 2 + TOKEN_LAYER_BYTES)
        self.decode_bytes = L * B * T * TOKEN_LAYER_BYTES + L * B * QO_BYTES_PER_SEQ_LAYER
        torch.cuda.synchronize()

    def append(self):
        self.kvq.quantize_append(self.shape, self.calib, self.cache, self.k, self.v, self.slots)

    def decode(self):
        self.kvq.decode_attention(self.shape, self.calib, self.cache, self.q, self.pt, self.seq_lens, out=self.out,
                                  workspace=self.ws)


def nvtx(name: str):
    """An NVTX range (for filtering a profiler capture to the timed steps)."""
    return torch.cuda.nvtx.range(name)


def time_two_kernels(first, second, warmup: int, steps: int, world: int):
    """Time steps of first() + second() with events around each call."""
    st = torch.cuda.current_stream()
    with nvtx("warmup"):
        for _ in range(warmup):
            first()
            second()
    torch.cuda.synchronize()
    barrier(world)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(st)
    with nvtx("timed steps"):
        for i in range(steps):
            ev[i][0].record(st)
            first()
            ev[i][1].record(st)
            second()
            ev[i][2].record(st)
    t1.record(st)
    torch.cuda.synchronize()
    barrier(world)
    return (t0.elapsed_time(t1), [e[0].elapsed_time(e[1]) for e in ev], [e[1].elapsed_time(e[2]) for e in ev])


def time_device(wl: Ragged, warmup: int, steps: int, world: int):
    st = torch.cuda.current_stream()
    with nvtx("warmup"):
        for i in range(warmup):
            s = i % wl.S
            wl.append(s)
            wl.decode(s)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dec_bytes = 0
    t0.record(st)
    with nvtx("timed steps"):
        for i in range(steps):
            s = (warmup + i) % wl.S
            with nvtx(f"step {i}: append"):
                wl.append(s)
            ev[i][0].record(st)
            with nvtx(f"step {i}: decode"):
                wl.decode(s)
            ev[i][1].record(st)
            dec_bytes += wl.decode_bytes(s)
    t1.record(st)
    torch.cuda.synchronize()
    barrier(world)
    total_ms = t0.elapsed_time(t1)
    dec_ms = [a.elapsed_time(b) for a, b in ev]
    return total_ms, dec_ms, dec_bytes / steps


def time_e2e(wl: Ragged, steps: int, world: int):
    """Same steps through the public API from pinned host buffers, copies inside.

    Every step copies its own query, new K/V and slots in and its output out.
    The copies run on a second stream into double-buffered device buffers, so
    step i+1's inputs move while step i computes (as a serving loop would).
    """
    st = torch.cuda.current_stream()
    cp = torch.cuda.Stream()
    S = wl.S
    n_host = min(S, steps)
    hq = wl.q[:n_host].cpu().pin_memory()
    hk = wl.k_new[:n_host].cpu().pin_memory()
    hv = wl.v_new[:n_host].cpu().pin_memory()
    hslots = wl.slots.cpu().pin_memory()
    hlens = wl.seq_lens.cpu().pin_memory()
    hout = [torch.empty(wl.out.shape, dtype=wl.out.dtype).pin_memory() for _ in range(2)]
    dq = [torch.empty_like(wl.q[0]) for _ in range(2)]
    dk = [torch.empty_like(wl.k_new[0]) for _ in range(2)]
    dv = [torch.empty_like(wl.v_new[0]) for _ in range(2)]
    dslots = [torch.empty_like(wl.slots[0]) for _ in range(2)]
    dlens = [torch.empty_like(wl.seq_lens[0]) for _ in range(2)]
    dout = [torch.empty_like(wl.out) for _ in range(2)]
    h2d = hq[0].numel() * 2 + hk[0].numel() * 2 * 2 + hslots[0].numel() * 8 + hlens[0].numel() * 4
    d2h = hout[0].numel() * 2
    ready = [torch.cuda.Event() for _ in range(2)]
    done = [torch.cuda.Event() for _ in range(2)]
    freed = [torch.cuda.Event() for _ in range(2)]
    torch.cuda.synchronize()
    barrier(world)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(st)
    cp.wait_stream(st)

    def h2d_step(i):
        j, s = i % 2, i % n_host
        with torch.cuda.stream(cp):
            if i >= 2:
                cp.wait_event(freed[j])
            dq[j].copy_(hq[s], non_blocking=True)
            dk[j].copy_(hk[s], non_blocking=True)
            dv[j].copy_(hv[s], non_blocking=True)
            dslots[j].copy_(hslots[s], non_blocking=True)
            dlens[j].copy_(hlens[s], non_blocking=True)
            ready[j].record(cp)

    h2d_step(0)
    for i in range(steps):
        j = i % 2
        if i + 1 < steps:
            h2d_step(i + 1)
        st.wait_event(ready[j])
        wl.kvq.quantize_append(wl.shape, wl.calib, wl.cache, dk[j], dv[j], dslots[j])
        wl.kvq.decode_attention(wl.shape, wl.calib, wl.cache, dq[j], wl.page_table_dev, dlens[j], out=dout[j],
                                workspace=wl.ws)
        freed[j].record(st)
        done[j].record(st)
        with torch.cuda.stream(cp):
            cp.wait_event(done[j])
            hout[j].copy_(dout[j], non_blocking=True)
    st.wait_stream(cp)
    t1.record(st)
    torch.cuda.synchronize()
    barrier(world)
    return t0.elapsed_time(t1), h2d, d2h


# ------------------------------------------------------------------ CPU oracle
def oracle_sample(seconds: float, layers=None):
    """Time the oracle on (layer, sequence) units of a ragged decode step until
    `seconds` pass; returns (tokens/s extrapolated to the full step, sample text)."""
    import oracle
    import synth
    w = synth.WORKLOADS["ragged"]
    lens = synth.ragged_lengths(w)
    units = [(l, b) for l in (layers or range(w.num_layers)) for b in range(w.batch)]
    done_tok_layers = 0
    spent = 0.0
    n_units = 0
    cal_cache = {}
    for (l, b) in units:
        if spent >= seconds:
            break
        if l not in cal_cache:
            kc, vc = synth.calibration_windows(w, l)
            cal_cache[l] = oracle.calibrate(kc[None], vc[None], exclude_pos0=True)
        s, inv, gk, gv = cal_cache[l]
        n = int(lens[b]) + 1
        k, v = synth.sequence_kv(w, l, b, n)
        q = synth.decode_queries(w, l, 0)[b][None]
        k32, v32, q32 = k.float().numpy(), v.float().numpy(), q.float().numpy()
        t = time.perf_counter()
        oracle.decode_reference(q32, k32, v32, s[0], inv[0], gk[0], gv[0])
        spent += time.perf_counter() - t
        done_tok_layers += n
        n_units += 1
    full_tok_layers = (int(lens.sum()) + w.batch) * w.num_layers
    step_s = spent / done_tok_layers * full_tok_layers
    sample = (f"{n_units} (layer, sequence) units of a ragged decode step ({done_tok_layers} token-layers, "
              f"{spent:.1f} s), extrapolated linearly to all 36 layers x 64 sequences")
    return w.batch / step_s, sample, spent


def cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


# ------------------------------------------------------------------ main
def config_block(wl=None):
    layers = wl.L if wl is not None else 36
    bf16k = wl is not None and wl.k_format == 1
    return {"workload": f"ragged decode: {layers} layers, 32 q / 8 kv heads, head_dim 128, batch 64, "
                        "lengths U[1024,8192], 16-token pages in shuffled order, 64 append+decode steps cycled",
            "batch": 64, "layers": layers,
            "kv_cache": ("mixed: bf16 keys, nvfp4 values" if bf16k else
                         "nvfp4 (e2m1 codes, e4m3 per-16 scales, fp32 tensor scale)" +
                         (", keys smoothed then rotated by a static per-head KLT" if wl is not None and wl.klt else "")),
            "l2": "inputs larger than L2 (about %.1f GB of cache read per step)" % (
                (28.2 if bf16k else 12.4) * layers / 36),
            "parallelism": "replicas (independent sequences per GPU)"}


def tensor_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            pk = json.load(f)
        return (float(pk["bf16_tflops"]), float(pk.get("bf16_tflops_sustained", pk["bf16_tflops"])),
                "measured (cuBLAS bf16 burst; fp16 runs at the same rate)")
    except (OSError, KeyError, ValueError):
        return 1590.0, 1400.0, "fallback"


def measure_prefill(kvq, synth, layers, k_format, qk_fp4, warm, steps, world):
    """Chunked causal prefill: per-step times of the chunk append and of the
    prefill launch, and the prefill kernel's roofline entry."""
    wl = Prefill(kvq, synth, layers, k_format=k_format, qk_fp4=qk_fp4)
    total, app_ms, pre_ms = time_two_kernels(wl.append, wl.attend, warm, steps, world)
    peak_tf, peak_tf_sus, tf_kind = tensor_peaks()
    pre = statistics.mean(pre_ms)
    achieved = wl.flops / (pre / 1e3) / 1e12
    if qk_fp4:
        # half the algorithmic flops (Q.K) run on FP4 operands at 4x the bf16 rate
        # (nominal 9 vs 2.25 PFLOP/s dense), half (P.V) on fp16 at the bf16 rate:
        # the mix's peak is 2 / (1/4 + 1) = 1.6x the bf16 one
        peak_tf, peak_tf_sus = 1.6 * peak_tf, 1.6 * peak_tf_sus
        tf_kind += "; x1.6 for the FP4 Q.K / fp16 P.V mix (FP4 = 4x bf16, nominal ratio)"
    roof = {"bound": "tensor", "achieved": achieved, "peak": peak_tf, "unit": "TFLOP/s",
            "frac": achieved / peak_tf, "frac_of_sustained": achieved / peak_tf_sus, "traffic": None,
            "peak_source": tf_kind,
            "kernel": "kvq prefill fp4 Q.K (tcgen05 mxf4nvf4 + f16)" if qk_fp4 else "kvq prefill (tcgen05)",
            "alg_flops_per_launch": wl.flops,
            "note": "algorithmic flops count 4 per attended (query head, key, dim)" +
                    ("" if qk_fp4 else "; the kernel issues 1.5x that on the tensor pipe (query hi + lo)")}
    out = {"total_ms": total, "append_ms": statistics.mean(app_ms), "prefill_ms": pre, "roofline": roof,
           "tokens": wl.B * wl.Tq * steps, "L": wl.L, "k_format": wl.k_format}
    del wl
    torch.cuda.empty_cache()
    return out


def measure_prefix(kvq, synth, name, layers, warm, steps, world):
    """Prefix workload (qwen3_8b or hadamard): per-step times of the bulk
    append of every layer's prefix and of one decode step of every layer."""
    wl = Prefix(kvq, synth, name, layers)
    total, app_ms, dec_ms = time_two_kernels(wl.append, wl.decode, warm, steps, world)
    peak_hbm, hbm_kind = measured_peak()
    app, dec = statistics.mean(app_ms), statistics.mean(dec_ms)
    out = {"total_ms": total, "append_ms": app, "decode_ms": dec, "B": wl.B, "T": wl.T, "L": wl.L,
           "hadamard": wl.w.hadamard, "launches": wl.launches,
           "decode": {"achieved": wl.decode_bytes / (dec / 1e3) / 1e9, "peak": peak_hbm, "unit": "GB/s",
                      "frac": wl.decode_bytes / (dec / 1e3) / 1e9 / peak_hbm, "peak_source": hbm_kind,
                      "alg_bytes_per_launch": wl.decode_bytes, "ms": dec},
           "append": {"achieved": wl.append_bytes / (app / 1e3) / 1e9, "unit": "GB/s",
                      "frac": wl.append_bytes / (app / 1e3) / 1e9 / peak_hbm,
                      "alg_bytes_per_launch": wl.append_bytes, "ms": app}}
    del wl
    torch.cuda.empty_cache()
    return out


PREFILL_METRIC = "NVFP4-KV chunked causal prefill tokens/s; achieved tensor TFLOP/s vs B200 peak"
PREFILL_WORKLOAD = ("chunked prefill: {L} layers, batch 8, 8192 cached + 512-token causal chunk, 32 q / 8 kv "
                    "heads, head_dim 128")
PREFIX_WORKLOAD = "{name}: {L} layers, batch {B} x {T} tokens; one step = quantise-append of the whole prefix + " \
                  "one decode step"


def other_workload(args, kvq, synth, rank, world):
    """One JSON line for the chunked-prefill or prefix workloads."""
    warm = max(3, args.warmup)
    clock = ClockSampler(torch.cuda.current_device()) if rank == 0 else None
    if args.workload == "prefill":
        qk_fp4 = args.qk == "fp4"
        r = measure_prefill(kvq, synth, args.layers, 1 if args.k_format == "bf16" else 0, qk_fp4, warm,
                            args.steps, world)
        clocks = clock.stop() if clock else None
        total = max_over_ranks(r["total_ms"], world)
        line = {"metric": PREFILL_METRIC, "value": world * r["tokens"] / (total / 1e3), "unit": "tokens/s",
                "n_gpus": world, "steps": args.steps, "warmup": warm, "ms_per_step": total / args.steps,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "data": "synthetic",
                "dtype": (PREFILL_DTYPE_FP4 if qk_fp4 else PREFILL_DTYPE_F16),
                "config": {"workload": PREFILL_WORKLOAD.format(L=r["L"]), "layers": r["L"],
                           "kv_cache": "mixed: bf16 keys, nvfp4 values" if r["k_format"] else "nvfp4",
                           "qk": "fp4" if qk_fp4 else "fp16"},
                "roofline": r["roofline"], "append_ms": r["append_ms"], "prefill_ms": r["prefill_ms"],
                "gpu_launches": 2 * args.steps, "clocks": clocks}
    else:
        r = measure_prefix(kvq, synth, args.workload, args.layers, warm, args.steps, world)
        clocks = clock.stop() if clock else None
        total = max_over_ranks(r["total_ms"], world)
        roof = dict(r["decode"], bound="hbm", traffic=None, kernel="kvq decode (split merge fused)")
        line = {"metric": METRIC, "value": world * r["B"] * args.steps / (total / 1e3), "unit": "tokens/s",
                "n_gpus": world, "steps": args.steps, "warmup": warm, "ms_per_step": total / args.steps,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": DECODE_DTYPE,
                "data": "synthetic",
                "config": {"workload": PREFIX_WORKLOAD.format(name=args.workload, L=r["L"], B=r["B"], T=r["T"]),
                           "hadamard": r["hadamard"]},
                "roofline": roof, "append": r["append"], "decode_ms": r["decode_ms"],
                "gpu_launches": r["launches"] * args.steps, "clocks": clocks}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def secondary_workloads(kvq, synth, warm=3, steps=5, prefix_steps=20):
    """The other workloads' kernel numbers, measured in the same run as the
    headline (each with its own clock samples), so they sit on the record
    beside it: the chunked prefill with fp16 and with FP4 Q.K (36 layers,
    batch 8, 8192 + 512 tokens) and the qwen3_8b and hadamard prefix
    workloads (bulk append + one decode step).  Each workload is freed before
    the next one is built.  The prefix workloads' decode launches are short
    (qwen3_8b: about 82 us) against the coarse grid CUDA event times fall on
    here (about 2 us), so they are averaged over more steps."""
    out = {}
    for key, qk_fp4 in (("prefill_fp16_qk", False), ("prefill_fp4_qk", True)):
        clock = ClockSampler(torch.cuda.current_device())
        r = measure_prefill(kvq, synth, 36, 0, qk_fp4, warm, steps, 1)
        roof = r["roofline"]
        out[key] = {"workload": PREFILL_WORKLOAD.format(L=r["L"]), "steps": steps, "warmup": warm,
                    "prefill_ms": r["prefill_ms"], "append_ms": r["append_ms"],
                    "tflops": roof["achieved"], "peak": roof["peak"], "frac": roof["frac"],
                    "frac_of_sustained": roof["frac_of_sustained"], "peak_source": roof["peak_source"],
                    "dtype": PREFILL_DTYPE_FP4 if qk_fp4 else PREFILL_DTYPE_F16, "clocks": clock.stop()}
    for name in ("qwen3_8b", "hadamard"):
        clock = ClockSampler(torch.cuda.current_device())
        r = measure_prefix(kvq, synth, name, 36, warm, prefix_steps, 1)
        out[name] = {"workload": PREFIX_WORKLOAD.format(name=name, L=r["L"], B=r["B"], T=r["T"]),
                     "steps": prefix_steps, "warmup": warm,
                     "decode": {k: r["decode"][k] for k in ("ms", "achieved", "frac", "unit")},
                     "append": {k: r["append"][k] for k in ("ms", "achieved", "frac", "unit")},
                     "clocks": clock.stop()}
    return out


def main():
    args = parse()
    if args.source_sha:
        print(decode_source_sha())
        return
    rank, world, local = dist_setup(args)
    if args.impl == "reference":
        if rank != 0:
            return
        # each step: one bounded sample of the workload -- the oracle on
        # (layer, sequence) units of one layer of a ragged decode step
        vals, spent = [], []
        sample = ""
        for i in range(args.warmup + args.steps):
            v, sample, sp = oracle_sample(max(1.0, args.cpu_seconds / 4), layers=[i % 36])
            if i >= args.warmup:
                vals.append(v)
                spent.append(sp)
        value = statistics.median(vals)
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": statistics.mean(spent) * 1e3, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64 (fp32 quantiser, fp64 attention)",
                "data": "synthetic", "config": config_block(), "impl": "reference",
                "step": "one bounded sample: the oracle on (layer, sequence) units of one layer of a ragged "
                        "decode step; value = its token-layer rate expressed as tokens/s of the whole step",
                "full_step_ms_extrapolated": 64 / value * 1e3,
                "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores(), "kind": "oracle",
                                 "sample": "per step: " + sample},
                "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    import bit_attention_decode_b200 as kvq
    import synth
    assert torch.cuda.is_available(), "bench needs a CUDA device"
    if args.workload != "ragged":
        return other_workload(args, kvq, synth, rank, world)
    t_setup = time.time()
    wl = Ragged(kvq, synth, args.layers, k_format=1 if args.k_format == "bf16" else 0, klt=args.klt)
    sys.stderr.write(f"[bench] setup {time.time() - t_setup:.1f} s, {wl.num_pages} pages, "
                     f"cache {wl.cache.data.numel() / 1e9:.2f} GB\n")
    clock = ClockSampler(torch.cuda.current_device()) if rank == 0 else None
    wl.time_bulk_append()
    total_ms, dec_ms, dec_bytes = time_device(wl, max(3, args.warmup), args.steps, world)
    clocks = clock.stop() if clock else None
    total_ms = max_over_ranks(total_ms, world)
    value = world * wl.B * args.steps / (total_ms / 1e3)
    dec_avg_ms = statistics.mean(dec_ms)
    achieved = dec_bytes / (dec_avg_ms / 1e3) / 1e9
    peak, peak_kind = measured_peak()
    # the committed ncu counters are those of the packed-key kernel
    traffic = ncu_traffic() if wl.k_format == 0 and not wl.klt else None
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": max(3, args.warmup), "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": DECODE_DTYPE, "data": "synthetic",
            "config": config_block(wl),
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": traffic, "peak_source": peak_kind,
                         "kernel": "kvq decode (split merge fused)", "alg_bytes_per_launch": dec_bytes},
            "append": append_entry(wl, peak),
            "gpu_launches": wl.launches_per_step * args.steps,
            "clocks": clocks}
    if not args.no_e2e:
        e_ms, h2d, d2h = time_e2e(wl, args.steps, world)
        e_ms = max_over_ranks(e_ms, world)
        line["e2e"] = {"value": world * wl.B * args.steps / (e_ms / 1e3), "unit": "tokens/s",
                       "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    del wl
    torch.cuda.empty_cache()
    if world == 1 and not args.no_secondary:
        line["secondary"] = secondary_workloads(kvq, synth)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, sample, _ = oracle_sample(args.cpu_seconds)
        line["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": cores(), "kind": "oracle",
                                "sample": sample}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
