"""Seeded synthetic inputs for the NVFP4 attention cache.

This module is the one piece shared by the tests, the bench and the smoke run:
it draws keys, values, queries, calibration windows, ragged lengths and page
tables.  It holds no step of the quantisation or attention method itself -- both
the CPU oracle and the CUDA library receive the tensors it returns as inputs.

Recipe (stated once, used by every workload):

* Model statistics per (layer, kv head): channel std ``sigma_c = exp(N(0, 1))``
  for the 128 channels of head_dim, and 4 channels drawn at random get
  ``sigma x 20`` (outlier channels).
* Pre-RoPE keys ``k[t, c] = sigma_c * N(0, 1)``; the token at position 0 of a
  sequence or calibration window is an attention sink whose key is scaled x40.
  The comment thread on GPTQ for NVFP4 weights (rstation.ai, krylov_schur)
  reports attention-sink token norms of 30-50x the typical token.
* Keys are rotated with NeoX rotate-half RoPE, ``theta = 1e6``, at their
  absolute position, so the cache holds post-RoPE keys as in the setup
  paragraph of "NVFP4 attention cache on W4A4 Qwen3-8B" (rstation.ai).
* Values and queries are ``N(0, 1)``; queries are taken as already post-RoPE.
* Tensors are rounded to bf16 (fp32 for the tiny workload).

Every draw comes from its own ``torch.Generator`` seeded from
``(workload seed, stream, layer, item)``, so any one sequence of any layer can
be regenerated alone.  The CPU and CUDA generators give different streams for
the same seed; a test that compares against the oracle hands the oracle a host
copy of exactly the tensor the library saw.
"""

from __future__ import annotations

import dataclasses
from typing import Optional

import torch

__all__ = [
    "Workload", "WORKLOADS", "model_sigma", "sequence_kv", "calibration_windows",
    "decode_queries", "prefill_queries", "ragged_lengths", "build_page_table",
    "slot_mapping", "rope_tables",
]

# stream identifiers (part of the seed derivation)
_S_MODEL, _S_CACHE, _S_CALIB, _S_QUERY, _S_LENS, _S_PAGES, _S_PREFQ = 1, 2, 3, 4, 5, 6, 7

ROPE_THETA = 1.0e6
SINK_SCALE = 40.0
OUTLIER_SCALE = 20.0
NUM_OUTLIERS = 4


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shapes of one synthetic workload (see the module docstring for values)."""
    name: str
    index: int
    num_layers: int
    batch: int
    context: int                  # cached tokens per sequence (fixed lengths)
    ragged: Optional[tuple] = None  # (lo, hi) inclusive uniform lengths instead
    decode_steps: int = 1
    prefill_chunk: int = 0        # query chunk length of a chunked prefill
    calib_windows: int = 4
    calib_len: int = 512
    calib_from_cache: bool = False  # tiny: calibrate on the cached keys themselves
    hadamard: bool = False
    dtype: torch.dtype = torch.bfloat16
    num_q_heads: int = 32
    num_kv_heads: int = 8
    head_dim: int = 128
    page_size: int = 16

    @property
    def seed(self) -> int:
        return 1000 + self.index

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads


WORKLOADS = {
    # 1 layer, batch 1, 256 cached tokens, fp32; calibration on the same keys
    "tiny": Workload("tiny", 1, num_layers=1, batch=1, context=256,
                     calib_windows=1, calib_len=256, calib_from_cache=True,
                     dtype=torch.float32),
    # Qwen3-8B-shaped cache: 36 layers, batch 4 x 2304 tokens, bf16
    "qwen3_8b": Workload("qwen3_8b", 2, num_layers=36, batch=4, context=2304),
    # normalised Hadamard-128 after smoothing, batch 16 x 4096 tokens
    "hadamard": Workload("hadamard", 3, num_layers=36, batch=16, context=4096,
                         hadamard=True),
    # ragged decode: batch 64, lengths U{1024..8192}, 64 append+decode steps
    "ragged": Workload("ragged", 4, num_layers=36, batch=64, context=0,
                       ragged=(1024, 8192), decode_steps=64),
    # chunked causal prefill: 8192 cached + a 512-token chunk, batch 8
    "prefill": Workload("prefill", 5, num_layers=36, batch=8, context=8192,
                        decode_steps=0, prefill_chunk=512),
}


def _gen(w: Workload, stream: int, layer: int, item: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((w.seed * 1_000_003 + stream * 100_003 + layer * 1_009 + item) % (2 ** 63))
    return g


def model_sigma(w: Workload, layer: int, device="cpu") -> torch.Tensor:
    """Per-channel key std [Hkv][D] (fp32) of one layer's synthetic model."""
    g = _gen(w, _S_MODEL, layer, 0, "cpu")
    sig = torch.exp(torch.randn(w.num_kv_heads, w.head_dim, generator=g, dtype=torch.float64))
    for h in range(w.num_kv_heads):
        idx = torch.randperm(w.head_dim, generator=g)[:NUM_OUTLIERS]
        sig[h, idx] *= OUTLIER_SCALE
    return sig.to(torch.float32).to(device)


def rope_tables(positions: torch.Tensor, head_dim: int):
    """cos/sin [n][D/2] (fp32) of NeoX RoPE at integer positions (theta 1e6)."""
    half = head_dim // 2
    inv = ROPE_THETA ** (-torch.arange(half, dtype=torch.float64) * 2.0 / head_dim)
    ang = positions.to(torch.float64).cpu()[:, None] * inv[None, :]
    return torch.cos(ang).to(torch.float32), torch.sin(ang).to(torch.float32)


def _rope(k: torch.Tensor, pos0: int) -> torch.Tensor:
    n, _, d = k.shape
    cos, sin = rope_tables(torch.arange(pos0, pos0 + n), d)
    cos = cos.to(k.device)[:, None, :]
    sin = sin.to(k.device)[:, None, :]
    a, b = k[..., : d // 2], k[..., d // 2:]
    return torch.cat([a * cos - b * sin, b * cos + a * sin], dim=-1)


def _draw_kv(w: Workload, sigma: torch.Tensor, n: int, pos0: int, g: torch.Generator, device):
    shape = (n, w.num_kv_heads, w.head_dim)
    k = torch.randn(shape, generator=g, device=device, dtype=torch.float32) * sigma.to(device)[None]
    v = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if pos0 == 0 and n > 0:
        k[0] *= SINK_SCALE
    k = _rope(k, pos0)
    return k.to(w.dtype), v.to(w.dtype)


def sequence_kv(w: Workload, layer: int, seq: int, n_tokens: int, device="cpu"):
    """Post-RoPE K and V [n_tokens][Hkv][D] of one sequence (positions 0..n-1).

    The tokens a ragged or prefill workload appends later are the tail of this
    same draw, so a sequence is one deterministic stream of tokens.
    """
    sigma = model_sigma(w, layer)
    return _draw_kv(w, sigma, n_tokens, 0, _gen(w, _S_CACHE, layer, seq, device), device)


def calibration_windows(w: Workload, layer: int, device="cpu"):
    """Calibration keys and values [W][T][Hkv][D] of one layer.

    Each window is a separate sequence starting at position 0 (a sink).  The
    tiny workload calibrates on its own cached keys (one window).
    """
    if w.calib_from_cache:
        k, v = sequence_kv(w, layer, 0, w.calib_len, device)
        return k[None], v[None]
    sigma = model_sigma(w, layer)
    ks, vs = [], []
    for win in range(w.calib_windows):
        k, v = _draw_kv(w, sigma, w.calib_len, 0, _gen(w, _S_CALIB, layer, win, device), device)
        ks.append(k)
        vs.append(v)
    return torch.stack(ks), torch.stack(vs)


def decode_queries(w: Workload, layer: int, step: int, device="cpu") -> torch.Tensor:
    """Decode queries [B][Hq][D] of one layer and step, N(0, 1)."""
    g = _gen(w, _S_QUERY, layer, step, device)
    q = torch.randn((w.batch, w.num_q_heads, w.head_dim), generator=g, device=device)
    return q.to(w.dtype)


def prefill_queries(w: Workload, layer: int, device="cpu") -> torch.Tensor:
    """Prefill query chunk [B][Tq][Hq][D] of one layer, N(0, 1)."""
    g = _gen(w, _S_PREFQ, layer, 0, device)
    q = torch.randn((w.batch, w.prefill_chunk, w.num_q_heads, w.head_dim), generator=g, device=device)
    return q.to(w.dtype)


def ragged_lengths(w: Workload) -> torch.Tensor:
    """Cached length per sequence [B] (int32): fixed, or uniform on [lo, hi]."""
    if w.ragged is None:
        return torch.full((w.batch,), w.context, dtype=torch.int32)
    lo, hi = w.ragged
    g = _gen(w, _S_LENS, 0, 0, "cpu")
    return torch.randint(lo, hi + 1, (w.batch,), generator=g, dtype=torch.int64).to(torch.int32)


def build_page_table(w: Workload, capacity: torch.Tensor, shuffle: bool = True, extra_pages: int = 0):
    """Page table [B][max_pages] int32 for sequences of the given token capacity.

    Pages are ``page_size``-token blocks of one shared pool.  With ``shuffle``
    the pool's page ids are handed out in a seeded random permutation, so the
    pages of a sequence are scattered over the pool.  Unused entries are -1.
    Returns (page_table, num_pages).
    """
    P = w.page_size
    npages = [(int(c) + P - 1) // P for c in capacity.tolist()]
    total = sum(npages) + extra_pages
    if shuffle:
        perm = torch.randperm(total, generator=_gen(w, _S_PAGES, 0, 0, "cpu")).to(torch.int32)
    else:
        perm = torch.arange(total, dtype=torch.int32)
    maxp = max(npages) if npages else 0
    table = torch.full((len(npages), max(maxp, 1)), -1, dtype=torch.int32)
    off = 0
    for b, n in enumerate(npages):
        table[b, :n] = perm[off:off + n]
        off += n
    return table, total


def slot_mapping(page_table: torch.Tensor, seq: torch.Tensor, pos: torch.Tensor, page_size: int = 16):
    """Cache slot (page * page_size + offset) of token ``pos`` of sequence ``seq``."""
    seq = seq.to(torch.int64)
    pos = pos.to(torch.int64)
    page = page_table.to(torch.int64)[seq, pos // page_size]
    return page * page_size + pos % page_size
