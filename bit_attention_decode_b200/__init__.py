"""NVFP4 attention cache for B200 -- Python binding of the kvq C ABI.

Argument marshalling only: every step of calibration, quantise-append and
attention runs in the CUDA kernels of ``libkvq.so`` (declared in
``include/kvq.h``).  PyTorch supplies device memory and the current stream.
There is no CPU fallback: if the library is missing, importing this package
raises ``ImportError``; build it with ``python bit_attention_decode_b200/build.py``.
"""

from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libkvq.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python bit_attention_decode_b200/build.py`")

_lib = ctypes.CDLL(LIB_PATH)

HEAD_DIM = 128
PAGE_SIZE = 16
TILE_BYTES = 2304

KVQ_OK, KVQ_EINVAL, KVQ_ECUDA, KVQ_EUNSUPPORTED, KVQ_EWORKSPACE = 0, 1, 2, 3, 4
DEV_BAD_PAGE, DEV_BAD_SLOT, DEV_BAD_LEN, DEV_TIMEOUT, DEV_BAD_WORKSPACE = 1, 2, 4, 8, 16
KVQ_F32, KVQ_BF16 = 0, 1
K_NVFP4, K_BF16 = 0, 1          # kvq_shape.k_format: packed keys, or bf16 keys (mixed cache)


class _Shape(ctypes.Structure):
    _fields_ = [("num_layers", ctypes.c_int32), ("num_q_heads", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("page_size", ctypes.c_int32), ("use_hadamard", ctypes.c_int32), ("k_format", ctypes.c_int32),
                ("use_klt", ctypes.c_int32)]


class _Calib(ctypes.Structure):
    _fields_ = [("k_smooth", ctypes.c_void_p), ("k_inv_smooth", ctypes.c_void_p),
                ("k_gscale", ctypes.c_void_p), ("v_gscale", ctypes.c_void_p), ("k_klt", ctypes.c_void_p)]


class _Cache(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("layer_stride_bytes", ctypes.c_int64),
                ("num_pages", ctypes.c_int32)]


_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_SHP, _CAL, _CCH = ctypes.POINTER(_Shape), ctypes.POINTER(_Calib), ctypes.POINTER(_Cache)

_lib.kvq_page_bytes.restype = ctypes.c_size_t
_lib.kvq_page_bytes.argtypes = [_SHP]
_lib.kvq_status_string.restype = ctypes.c_char_p
_lib.kvq_status_string.argtypes = [_I32]
_lib.kvq_version.restype = ctypes.c_char_p
_lib.kvq_version.argtypes = []
_lib.kvq_calibrate_smoothing.restype = _I32
_lib.kvq_calibrate_smoothing.argtypes = [_SHP, _P, _P, _I32, _I32, _I32, _I32, _CAL, _P]
_lib.kvq_calibrate_klt.restype = _I32
_lib.kvq_calibrate_klt.argtypes = [_SHP, _P, _P, _I32, _I32, _I32, _I32, _CAL, _P]
_lib.kvq_calibrate_native.restype = _I32
_lib.kvq_calibrate_native.argtypes = [_SHP, _P, _P, _I32, _I32, _I32, _CAL, _P]
_lib.kvq_quantize_append.restype = _I32
_lib.kvq_quantize_append.argtypes = [_SHP, _CAL, _CCH, _I32, _I32, _P, _P, _I32, _P, _I32, _P, _P]
_lib.kvq_decode_workspace_bytes.restype = ctypes.c_size_t
_lib.kvq_decode_workspace_bytes.argtypes = [_SHP, _I32, _I32, _I32]
_lib.kvq_decode_attention.restype = _I32
_lib.kvq_decode_attention.argtypes = [_SHP, _CAL, _CCH, _I32, _I32, _P, _I32, _P, _I32, _P, _I32, _P, _I32,
                                      _P, ctypes.c_size_t, _P, _P]
_lib.kvq_prefill_workspace_bytes.restype = ctypes.c_size_t
_lib.kvq_prefill_workspace_bytes.argtypes = [_SHP, _I32, _I32, _I32]
_lib.kvq_prefill_attention.restype = _I32
_lib.kvq_prefill_attention.argtypes = [_SHP, _CAL, _CCH, _I32, _I32, _P, _I32, _I32, _P, _P, _I32, _P, _I32,
                                       _P, _I32, _P, ctypes.c_size_t, _P, _P]
_lib.kvq_prefill_attention_fp4.restype = _I32
_lib.kvq_prefill_attention_fp4.argtypes = _lib.kvq_prefill_attention.argtypes
_lib.kvq_decode_attention_noalloc.restype = _I32
_lib.kvq_decode_attention_noalloc.argtypes = [_SHP, _CAL, _CCH, _I32, _I32, _P, _I32, _P, _I32, _P, _I32, _P,
                                              _I32, _P, _P]
_lib.kvq_selftest_wait_timeout.restype = _I32
_lib.kvq_selftest_wait_timeout.argtypes = [_P, ctypes.c_int64, _P]
_lib.kvq_round_e2m1.restype = _I32
_lib.kvq_round_e2m1.argtypes = [_P, _P, ctypes.c_int64, _P]
_lib.kvq_round_e4m3.restype = _I32
_lib.kvq_round_e4m3.argtypes = [_P, _P, ctypes.c_int64, _P]

EXPORTED = ("kvq_page_bytes", "kvq_status_string", "kvq_version", "kvq_calibrate_smoothing", "kvq_calibrate_native",
            "kvq_calibrate_klt",
            "kvq_quantize_append", "kvq_decode_workspace_bytes", "kvq_decode_attention",
            "kvq_prefill_workspace_bytes", "kvq_prefill_attention", "kvq_prefill_attention_fp4",
            "kvq_decode_attention_noalloc",
            "kvq_round_e2m1", "kvq_round_e4m3", "kvq_selftest_wait_timeout")

NOALLOC_SCRATCH_BYTES = 16 << 20


class KVQError(RuntimeError):
    def __init__(self, status: int, call: str):
        super().__init__(f"{call}: {status_string(status)} (status {status})")
        self.status = status


def status_string(status: int) -> str:
    return _lib.kvq_status_string(int(status)).decode()


def version() -> str:
    return _lib.kvq_version().decode()


def _check(status: int, call: str):
    if status != KVQ_OK:
        raise KVQError(status, call)


@dataclasses.dataclass(frozen=True)
class Shape:
    num_layers: int
    num_q_heads: int = 32
    num_kv_heads: int = 8
    use_hadamard: bool = False
    head_dim: int = HEAD_DIM
    page_size: int = PAGE_SIZE
    k_format: int = K_NVFP4
    use_klt: bool = False

    def c(self) -> _Shape:
        return _Shape(self.num_layers, self.num_q_heads, self.num_kv_heads, self.head_dim,
                      self.page_size, int(self.use_hadamard), int(self.k_format), int(self.use_klt))


@dataclasses.dataclass
class Calibration:
    """Static smoothing factors and FP32 tensor scales (device fp32 tensors)."""
    k_smooth: torch.Tensor       # [L][Hkv][128]
    k_inv_smooth: torch.Tensor   # [L][Hkv][128]
    k_gscale: torch.Tensor       # [L]
    v_gscale: torch.Tensor       # [L]
    k_klt: Optional[torch.Tensor] = None   # [L][Hkv][128][128] KLT bases (use_klt shapes)

    def c(self) -> _Calib:
        return _Calib(self.k_smooth.data_ptr(), self.k_inv_smooth.data_ptr(),
                      self.k_gscale.data_ptr(), self.v_gscale.data_ptr(), _ptr(self.k_klt))


@dataclasses.dataclass
class PagedCache:
    """Packed NVFP4 cache: uint8 [L][num_pages][Hkv * 2304] on the device."""
    data: torch.Tensor

    @property
    def num_pages(self) -> int:
        return self.data.shape[1]

    def c(self) -> _Cache:
        return _Cache(self.data.data_ptr(), self.data.stride(0), self.num_pages)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return KVQ_F32
    if t.dtype == torch.bfloat16:
        return KVQ_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _stream():
    return torch.cuda.current_stream().cuda_stream


def _need_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("kvq tensors must be contiguous CUDA tensors")


def page_bytes(shape: Shape) -> int:
    return int(_lib.kvq_page_bytes(ctypes.byref(shape.c())))


def new_calibration(shape: Shape, device="cuda") -> Calibration:
    L, H = shape.num_layers, shape.num_kv_heads
    f = dict(dtype=torch.float32, device=device)
    klt = torch.empty(L, H, HEAD_DIM, HEAD_DIM, **f) if shape.use_klt else None
    return Calibration(torch.empty(L, H, HEAD_DIM, **f), torch.empty(L, H, HEAD_DIM, **f),
                       torch.empty(L, **f), torch.empty(L, **f), klt)


def new_cache(shape: Shape, num_pages: int, device="cuda") -> PagedCache:
    return PagedCache(torch.zeros(shape.num_layers, num_pages, page_bytes(shape), dtype=torch.uint8, device=device))


def calibrate_smoothing(shape: Shape, k_calib: torch.Tensor, v_calib: torch.Tensor, exclude_pos0: bool = True,
                        out: Optional[Calibration] = None) -> Calibration:
    """k/v_calib [L][W][T][Hkv][128] post-RoPE calibration windows."""
    _need_cuda(k_calib, v_calib)
    L, W, T, H, D = k_calib.shape
    if out is None:
        out = new_calibration(shape, k_calib.device)
    c = out.c()
    _check(_lib.kvq_calibrate_smoothing(ctypes.byref(shape.c()), k_calib.data_ptr(), v_calib.data_ptr(),
                                        _dtype_code(k_calib), W, T, int(bool(exclude_pos0)), ctypes.byref(c),
                                        _stream()), "kvq_calibrate_smoothing")
    return out


def calibrate_native(shape: Shape, k_calib: torch.Tensor, v_calib: torch.Tensor,
                     out: Optional[Calibration] = None) -> Calibration:
    """Keys in their native basis (s = 1) with calibrated tensor scales;
    k/v_calib [L][W][T][Hkv][128]."""
    _need_cuda(k_calib, v_calib)
    L, W, T, H, D = k_calib.shape
    if out is None:
        out = new_calibration(shape, k_calib.device)
    c = out.c()
    _check(_lib.kvq_calibrate_native(ctypes.byref(shape.c()), k_calib.data_ptr(), v_calib.data_ptr(),
                                     _dtype_code(k_calib), W, T, ctypes.byref(c), _stream()),
           "kvq_calibrate_native")
    return out


def calibrate_klt(shape: Shape, k_calib: torch.Tensor, v_calib: torch.Tensor, exclude_pos0: bool = True,
                  out: Optional[Calibration] = None) -> Calibration:
    """Smoothing then a static per-head KLT (shape.use_klt);
    k/v_calib [L][W][T][Hkv][128]."""
    _need_cuda(k_calib, v_calib)
    L, W, T, H, D = k_calib.shape
    if out is None:
        out = new_calibration(shape, k_calib.device)
    c = out.c()
    _check(_lib.kvq_calibrate_klt(ctypes.byref(shape.c()), k_calib.data_ptr(), v_calib.data_ptr(),
                                  _dtype_code(k_calib), W, T, int(bool(exclude_pos0)), ctypes.byref(c), _stream()),
           "kvq_calibrate_klt")
    return out


def quantize_append(shape: Shape, calib: Calibration, cache: PagedCache, k: torch.Tensor, v: torch.Tensor,
                    slot_mapping: torch.Tensor, layer0: int = 0, status: Optional[torch.Tensor] = None):
    """k, v [nlayers][T][Hkv][128] (or [T][Hkv][128] for one layer); slot_mapping [T] int64."""
    if k.dim() == 3:
        k, v = k[None], v[None]
    _need_cuda(k, v, slot_mapping, status)
    assert slot_mapping.dtype == torch.int64
    nl, T = k.shape[0], k.shape[1]
    _check(_lib.kvq_quantize_append(ctypes.byref(shape.c()), ctypes.byref(calib.c()), ctypes.byref(cache.c()),
                                    layer0, nl, k.data_ptr(), v.data_ptr(), _dtype_code(k),
                                    slot_mapping.data_ptr(), T, _ptr(status), _stream()), "kvq_quantize_append")


def new_workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A workspace for decode_attention / prefill_attention: zero-filled, as
    the split merge's counters at its start must be before the first call
    (every call leaves them zero, so it can be reused for any later call)."""
    return torch.zeros(max(int(nbytes), 16), dtype=torch.uint8, device=device)


def decode_workspace_bytes(shape: Shape, nlayers: int, batch: int, max_pages_per_seq: int) -> int:
    return int(_lib.kvq_decode_workspace_bytes(ctypes.byref(shape.c()), nlayers, batch, max_pages_per_seq))


def decode_attention(shape: Shape, calib: Calibration, cache: PagedCache, q: torch.Tensor,
                     page_table: torch.Tensor, seq_lens: torch.Tensor, layer0: int = 0,
                     out: Optional[torch.Tensor] = None, out_dtype=torch.bfloat16,
                     workspace: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None):
    """q [nlayers][B][Hq][128] -> out [nlayers][B][Hq][128]."""
    if q.dim() == 3:
        q = q[None]
    nl, B = q.shape[0], q.shape[1]
    maxp = page_table.shape[1]
    if out is None:
        out = torch.empty(q.shape, dtype=out_dtype, device=q.device)
    need = decode_workspace_bytes(shape, nl, B, maxp)
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = new_workspace(need, q.device)
    _need_cuda(q, page_table, seq_lens, out, workspace, status)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.kvq_decode_attention(ctypes.byref(shape.c()), ctypes.byref(calib.c()), ctypes.byref(cache.c()),
                                     layer0, nl, q.data_ptr(), _dtype_code(q), page_table.data_ptr(), maxp,
                                     seq_lens.data_ptr(), B, out.data_ptr(), _dtype_code(out), _ptr(workspace),
                                     ws_bytes, _ptr(status), _stream()), "kvq_decode_attention")
    return out


def decode_attention_noalloc(shape: Shape, calib: Calibration, cache: PagedCache, q: torch.Tensor,
                             page_table: torch.Tensor, seq_lens: torch.Tensor, out: torch.Tensor,
                             layer0: int = 0, status: Optional[torch.Tensor] = None):
    """decode_attention with the library's static scratch array instead of a
    workspace: for callers that cannot allocate device memory.  ``out`` is
    required (this call allocates nothing); calls must not overlap on the GPU."""
    if q.dim() == 3:
        q = q[None]
    nl, B = q.shape[0], q.shape[1]
    _need_cuda(q, page_table, seq_lens, out, status)
    _check(_lib.kvq_decode_attention_noalloc(ctypes.byref(shape.c()), ctypes.byref(calib.c()),
                                             ctypes.byref(cache.c()), layer0, nl, q.data_ptr(), _dtype_code(q),
                                             page_table.data_ptr(), page_table.shape[1], seq_lens.data_ptr(), B,
                                             out.data_ptr(), _dtype_code(out), _ptr(status), _stream()),
           "kvq_decode_attention_noalloc")
    return out


def prefill_workspace_bytes(shape: Shape, nlayers: int, batch: int, q_len: int) -> int:
    return int(_lib.kvq_prefill_workspace_bytes(ctypes.byref(shape.c()), nlayers, batch, q_len))


def prefill_attention(shape: Shape, calib: Calibration, cache: PagedCache, q: torch.Tensor,
                      q_start: torch.Tensor, page_table: torch.Tensor, seq_lens: torch.Tensor, layer0: int = 0,
                      out: Optional[torch.Tensor] = None, out_dtype=torch.bfloat16,
                      workspace: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None,
                      qk_fp4: bool = False):
    """q [nlayers][B][q_len][Hq][128] -> out of the same shape.  qk_fp4:
    Q.K on the block-scaled FP4 tensor cores, the query quantised to NVFP4
    per row (kvq_prefill_attention_fp4)."""
    if q.dim() == 4:
        q = q[None]
    nl, B, Tq = q.shape[0], q.shape[1], q.shape[2]
    maxp = page_table.shape[1]
    if out is None:
        out = torch.empty(q.shape, dtype=out_dtype, device=q.device)
    need = prefill_workspace_bytes(shape, nl, B, Tq)
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = new_workspace(need, q.device)
    _need_cuda(q, q_start, page_table, seq_lens, out, workspace, status)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    name = "kvq_prefill_attention_fp4" if qk_fp4 else "kvq_prefill_attention"
    _check(getattr(_lib, name)(ctypes.byref(shape.c()), ctypes.byref(calib.c()), ctypes.byref(cache.c()),
                               layer0, nl, q.data_ptr(), _dtype_code(q), Tq, q_start.data_ptr(),
                               page_table.data_ptr(), maxp, seq_lens.data_ptr(), B, out.data_ptr(),
                               _dtype_code(out), _ptr(workspace), ws_bytes, _ptr(status), _stream()), name)
    return out


def selftest_wait_timeout(status: torch.Tensor, limit_ns: int = 20_000_000):
    """Run the bounded-wait self-test: ORs DEV_TIMEOUT into ``status`` (int32, device)."""
    _need_cuda(status)
    _check(_lib.kvq_selftest_wait_timeout(status.data_ptr(), int(limit_ns), _stream()), "kvq_selftest_wait_timeout")


def round_e2m1(x: torch.Tensor) -> torch.Tensor:
    """Elementwise fp32 -> E2M1 code (one per byte) with the kernels' rounding."""
    _need_cuda(x)
    out = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    _check(_lib.kvq_round_e2m1(x.data_ptr(), out.data_ptr(), x.numel(), _stream()), "kvq_round_e2m1")
    return out


def round_e4m3(x: torch.Tensor) -> torch.Tensor:
    """Elementwise fp32 -> E4M3 code with the kernels' rounding."""
    _need_cuda(x)
    out = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    _check(_lib.kvq_round_e4m3(x.data_ptr(), out.data_ptr(), x.numel(), _stream()), "kvq_round_e4m3")
    return out


def unpack_tiles(cache_layer: torch.Tensor, num_kv_heads: int):
    """Split a layer's cache bytes [num_pages][Hkv*2304] into its four fields.

    Returns (k_codes [P][H][16][64], k_scales [P][H][16][8],
    v_codes [P][H][16][64], v_scales [P][H][8][16]) as views; a reader for
    tests and tools, not part of any kernel path.
    """
    t = cache_layer.view(cache_layer.shape[0], num_kv_heads, TILE_BYTES)
    return (t[..., 0:1024].unflatten(-1, (16, 64)), t[..., 1024:1152].unflatten(-1, (16, 8)),
            t[..., 1152:2176].unflatten(-1, (16, 64)), t[..., 2176:2304].unflatten(-1, (8, 16)))
