"""Block-scaled tensor quantization on NVIDIA B200 (sm_100a).

A thin ctypes binding of libbq.so (C ABI in include/bq.h). The functions named
``bq_*`` marshal torch tensors (device memory) and the current CUDA stream into the
C entry points of the same names; every step of the computation runs in the CUDA
kernels. ``quantize`` / ``dequantize`` / ``qsnr`` add output allocation on top.

The library must be built (``python -m block_scaled_bit_bq_b200.build``); importing
this package without libbq.so raises, and there is no CPU fallback.
"""

from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbq.so")

# enums of include/bq.h
DT = {"bf16": 0, "fp16": 1, "fp32": 2, "ue8m0": 3, "e4m3": 4}
FORMATS = {"int8_sym": 0, "int8_asym": 1, "int4_sym": 2, "uint4_asym": 3, "e4m3": 4, "e5m2": 5, "e2m1": 6,
           "e2m3": 7, "e3m2": 8}
GRANULARITIES = {"tensor": 0, "row": 1, "group": 2, "mx": 3, "nv": 4, "tile2d": 5}
LAYOUTS = {"rows": 0, "gemm": 1}       # MX / NV block scales: row-major, or a block-scaled GEMM's tiles
FOUR_BIT = {"int4_sym", "uint4_asym", "e2m1"}
ASYMMETRIC = {"int8_asym", "uint4_asym"}

STATUS = {0: "BQ_OK", 1: "BQ_ERR_INVALID_ARG", 2: "BQ_ERR_UNSUPPORTED", 3: "BQ_ERR_SHAPE",
          4: "BQ_ERR_ALIGNMENT", 5: "BQ_ERR_WORKSPACE", 6: "BQ_ERR_CUDA"}


class BqError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {_lib().bq_status_string(status).decode()}")


class BqScheme(ctypes.Structure):
    _fields_ = [("format", ctypes.c_int32), ("granularity", ctypes.c_int32), ("block", ctypes.c_int32),
                ("scale_dtype", ctypes.c_int32), ("hadamard", ctypes.c_int32), ("scale_layout", ctypes.c_int32)]


class BqRowTransform(ctypes.Structure):
    _fields_ = [("col_scale", ctypes.c_void_p), ("sign_bits", ctypes.c_void_p), ("reserved", ctypes.c_int64)]


class BqStats(ctypes.Structure):
    _fields_ = [("err2", ctypes.c_double), ("x2", ctypes.c_double), ("kappa_sum", ctypes.c_double),
                ("kappa_max", ctypes.c_double), ("n_units", ctypes.c_double)]


_L = None


def _lib() -> ctypes.CDLL:
    global _L
    if _L is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m block_scaled_bit_bq_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
        sp = ctypes.POINTER(BqScheme)
        L.bq_status_string.restype = ctypes.c_char_p
        L.bq_status_string.argtypes = [ctypes.c_int]
        L.bq_version.restype = ctypes.c_char_p
        L.bq_version.argtypes = []
        L.bq_buffer_sizes.restype = ctypes.c_int
        L.bq_buffer_sizes.argtypes = [sp, i64, i64, ctypes.POINTER(sz), ctypes.POINTER(sz),
                                      ctypes.POINTER(sz), ctypes.POINTER(sz)]
        L.bq_workspace_size.restype = ctypes.c_int
        L.bq_workspace_size.argtypes = [sp, i64, i64, ctypes.c_int, ctypes.POINTER(sz)]
        L.bq_quantize.restype = ctypes.c_int
        L.bq_quantize.argtypes = [vp, i32, i64, i64, sp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.bq_dequantize.restype = ctypes.c_int
        L.bq_dequantize.argtypes = [vp, vp, vp, vp, i64, i64, sp, vp, i32, vp]
        L.bq_qsnr.restype = ctypes.c_int
        L.bq_qsnr.argtypes = [vp, i32, vp, vp, vp, vp, i64, i64, sp, vp, vp, sz, vp]
        L.bq_quantize_noalloc.restype = ctypes.c_int
        L.bq_quantize_noalloc.argtypes = [vp, i32, i64, i64, sp, vp, vp, vp, vp, vp, vp]
        L.bq_stats_qsnr_db.restype = ctypes.c_double
        L.bq_stats_qsnr_db.argtypes = [ctypes.POINTER(BqStats)]
        L.bq_stats_to_db.restype = ctypes.c_double
        L.bq_stats_to_db.argtypes = [ctypes.POINTER(BqStats)]
        L.bq_tensor_range.restype = ctypes.c_int
        L.bq_tensor_range.argtypes = [vp, i32, i64, i64, sp, vp, vp, sz, vp]
        L.bq_quantize_with_range.restype = ctypes.c_int
        L.bq_quantize_with_range.argtypes = [vp, i32, i64, i64, sp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.bq_quantize_batch.restype = ctypes.c_int
        L.bq_quantize_batch.argtypes = [vp, i32, i64, i64, i64, sp, vp, vp, vp, vp, vp, sz, vp]
        L.bq_gemm.restype = ctypes.c_int
        L.bq_gemm.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, sp, vp, i32, vp]
        L.bq_debug_skip_tile_copy.restype = ctypes.c_int
        L.bq_debug_skip_tile_copy.argtypes = [i32]
        L.bq_wait_timeouts.restype = ctypes.c_int
        L.bq_wait_timeouts.argtypes = [ctypes.POINTER(ctypes.c_uint32), i32]
        rtp = ctypes.POINTER(BqRowTransform)
        L.bq_quantize_rt.restype = ctypes.c_int
        L.bq_quantize_rt.argtypes = [vp, i32, i64, i64, sp, rtp, vp, vp, vp, vp, vp, sz, vp]
        L.bq_dequantize_rt.restype = ctypes.c_int
        L.bq_dequantize_rt.argtypes = [vp, vp, vp, i64, i64, sp, rtp, vp, i32, vp]
        _L = L
    return _L


def lib() -> ctypes.CDLL:
    """The loaded libbq.so (raises ImportError when it has not been built)."""
    return _lib()


@dataclass(frozen=True)
class Scheme:
    """A quantization scheme: element format, scaling granularity, group size, scale
    dtype, the Hadamard flag and the layout of MX / NV block scales ("rows", or "gemm":
    the tiles a block-scaled GEMM reads). block / scale_dtype default to the
    granularity's own (32 / ue8m0 for mx, 16 / e4m3 for nv, 128 / fp32 for tile2d
    (128 x 128 tiles), fp32 otherwise)."""
    fmt: str
    gran: str
    block: int = 0
    scale_dtype: str | None = None
    hadamard: bool = False
    layout: str = "rows"

    def resolved(self) -> "Scheme":
        sd = self.scale_dtype or {"mx": "ue8m0", "nv": "e4m3"}.get(self.gran, "fp32")
        blk = self.block or {"mx": 32, "nv": 16, "tile2d": 128}.get(self.gran, 0)
        return Scheme(self.fmt, self.gran, blk, sd, bool(self.hadamard), self.layout)

    def c(self) -> BqScheme:
        s = self.resolved()
        return BqScheme(FORMATS[s.fmt], GRANULARITIES[s.gran], s.block, DT[s.scale_dtype], int(s.hadamard),
                        LAYOUTS[s.layout])


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(status: int, where: str):
    if status != 0:
        raise BqError(status, where)


# ---------------------------------------------------------------------------
# C entry points (same names), tensor marshalling only
# ---------------------------------------------------------------------------

def bq_version() -> str:
    return _lib().bq_version().decode()


def bq_status_string(status: int) -> str:
    return _lib().bq_status_string(status).decode()


def bq_buffer_sizes(scheme: Scheme, rows: int, cols: int):
    """(code_bytes, scale_bytes, zero_point_bytes, tensor_scale_bytes)."""
    out = [ctypes.c_size_t(0) for _ in range(4)]
    sc = scheme.c()
    _check(_lib().bq_buffer_sizes(ctypes.byref(sc), rows, cols, *[ctypes.byref(o) for o in out]),
           "bq_buffer_sizes")
    return tuple(int(o.value) for o in out)


def bq_workspace_size(scheme: Scheme, rows: int, cols: int, with_stats: bool) -> int:
    out = ctypes.c_size_t(0)
    sc = scheme.c()
    _check(_lib().bq_workspace_size(ctypes.byref(sc), rows, cols, int(with_stats), ctypes.byref(out)),
           "bq_workspace_size")
    return int(out.value)


def bq_quantize(x: torch.Tensor, scheme: Scheme, codes: torch.Tensor, scales: torch.Tensor,
                zero_points: torch.Tensor | None, tensor_scale: torch.Tensor | None,
                stats: torch.Tensor | None, workspace: torch.Tensor | None, stream=None,
                rows: int | None = None, cols: int | None = None) -> None:
    """x: bf16 [rows, cols] on the device; outputs are preallocated device tensors."""
    if rows is None:
        rows, cols = x.shape
    sc = scheme.c()
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib().bq_quantize(_ptr(x), DT["bf16"], rows, cols, ctypes.byref(sc), _ptr(codes), _ptr(scales),
                              _ptr(zero_points), _ptr(tensor_scale), _ptr(stats), _ptr(workspace), ws_bytes,
                              _stream(stream)), "bq_quantize")


def bq_quantize_noalloc(x: torch.Tensor, scheme: Scheme, codes: torch.Tensor, scales: torch.Tensor,
                        zero_points: torch.Tensor | None, tensor_scale: torch.Tensor | None,
                        stats: torch.Tensor | None, stream=None) -> None:
    """bq_quantize with the library's own static device scratch instead of a workspace
    (for callers that cannot allocate device memory; calls must not overlap)."""
    rows, cols = x.shape
    sc = scheme.c()
    _check(_lib().bq_quantize_noalloc(_ptr(x), DT["bf16"], rows, cols, ctypes.byref(sc), _ptr(codes), _ptr(scales),
                                      _ptr(zero_points), _ptr(tensor_scale), _ptr(stats), _stream(stream)),
           "bq_quantize_noalloc")


def bq_tensor_range(x: torch.Tensor, scheme: Scheme, range_out: torch.Tensor, workspace: torch.Tensor,
                    stream=None) -> None:
    """The range pass of a per-tensor / NV scheme alone: range_out (fp32 [3] on the
    device) = {amax, min(min, 0), max(max, 0)} of the (rotated) tensor."""
    rows, cols = x.shape
    sc = scheme.c()
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(_lib().bq_tensor_range(_ptr(x), DT["bf16"], rows, cols, ctypes.byref(sc), _ptr(range_out),
                                  _ptr(workspace), ws_bytes, _stream(stream)), "bq_tensor_range")


def bq_quantize_with_range(x: torch.Tensor, scheme: Scheme, range_in: torch.Tensor, codes: torch.Tensor,
                           scales: torch.Tensor, zero_points: torch.Tensor | None,
                           tensor_scale: torch.Tensor | None, stats: torch.Tensor | None,
                           workspace: torch.Tensor | None, stream=None) -> None:
    """The quantize pass of a per-tensor / NV scheme against a given range (fp32 [3] on
    the device: amax, min, max)."""
    rows, cols = x.shape
    sc = scheme.c()
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib().bq_quantize_with_range(_ptr(x), DT["bf16"], rows, cols, ctypes.byref(sc), _ptr(range_in),
                                         _ptr(codes), _ptr(scales), _ptr(zero_points), _ptr(tensor_scale),
                                         _ptr(stats), _ptr(workspace), ws_bytes, _stream(stream)),
           "bq_quantize_with_range")


def bq_quantize_batch(x: torch.Tensor, scheme: Scheme, codes: torch.Tensor, scales: torch.Tensor,
                      zero_points: torch.Tensor | None, stats: torch.Tensor | None,
                      workspace: torch.Tensor | None, stream=None) -> None:
    """x: bf16 [batch, rows, cols] on the device; outputs preallocated (see alloc_batch_outputs);
    stats: float64 [batch, 5] or None."""
    batch, rows, cols = x.shape
    sc = scheme.c()
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib().bq_quantize_batch(_ptr(x), DT["bf16"], batch, rows, cols, ctypes.byref(sc), _ptr(codes),
                                    _ptr(scales), _ptr(zero_points), _ptr(stats), _ptr(workspace), ws_bytes,
                                    _stream(stream)), "bq_quantize_batch")


def bq_gemm(a: "Quantized", b: "Quantized", d: torch.Tensor, stream=None) -> None:
    """D[m, n] = A[m, k] B[n, k]^T on the tensor cores from two quantized operands (same
    MXFP8 or NVFP4 scheme, GEMM-layout scales); d: fp32 or bf16 [m, n] on the device."""
    if a.scheme != b.scheme or a.cols != b.cols:
        raise ValueError("operands need the same scheme and the same k")
    m, n, k = a.rows, b.rows, a.cols
    d_dt = {torch.bfloat16: DT["bf16"], torch.float32: DT["fp32"]}[d.dtype]
    sc = a.scheme.c()
    _check(_lib().bq_gemm(_ptr(a.codes), _ptr(a.scales), _ptr(a.tensor_scale), _ptr(b.codes), _ptr(b.scales),
                          _ptr(b.tensor_scale), m, n, k, ctypes.byref(sc), _ptr(d), d_dt, _stream(stream)), "bq_gemm")


def gemm(a: "Quantized", b: "Quantized", dtype=torch.float32, stream=None) -> torch.Tensor:
    """A B^T of two quantized operands (MXFP8 / NVFP4, GEMM-layout scales)."""
    d = torch.empty((a.rows, b.rows), dtype=dtype, device=a.codes.device)
    bq_gemm(a, b, d, stream)
    return d


def bq_debug_skip_tile_copy(warp: int) -> None:
    """Test hook: in the next flat quantize launch, warp `warp` issues no copy for its first
    staged tile, so its wait runs out (bounded) and bq_wait_timeouts counts it."""
    _check(_lib().bq_debug_skip_tile_copy(int(warp)), "bq_debug_skip_tile_copy")


def bq_dequantize(codes: torch.Tensor, scales: torch.Tensor, zero_points: torch.Tensor | None,
                  tensor_scale: torch.Tensor | None, rows: int, cols: int, scheme: Scheme,
                  out: torch.Tensor, stream=None) -> None:
    out_dt = {torch.bfloat16: DT["bf16"], torch.float32: DT["fp32"]}[out.dtype]
    sc = scheme.c()
    _check(_lib().bq_dequantize(_ptr(codes), _ptr(scales), _ptr(zero_points), _ptr(tensor_scale), rows, cols,
                                ctypes.byref(sc), _ptr(out), out_dt, _stream(stream)), "bq_dequantize")


def bq_qsnr(x: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor, zero_points: torch.Tensor | None,
            tensor_scale: torch.Tensor | None, scheme: Scheme, stats: torch.Tensor,
            workspace: torch.Tensor, stream=None) -> None:
    rows, cols = x.shape
    sc = scheme.c()
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(_lib().bq_qsnr(_ptr(x), DT["bf16"], _ptr(codes), _ptr(scales), _ptr(zero_points), _ptr(tensor_scale),
                          rows, cols, ctypes.byref(sc), _ptr(stats), _ptr(workspace), ws_bytes, _stream(stream)),
           "bq_qsnr")


def _rt(col_scale: torch.Tensor | None, sign_bits: torch.Tensor | None) -> BqRowTransform:
    return BqRowTransform(_ptr(col_scale), _ptr(sign_bits), 0)


def bq_quantize_rt(x: torch.Tensor, scheme: Scheme, col_scale: torch.Tensor | None, sign_bits: torch.Tensor | None,
                   codes: torch.Tensor, scales: torch.Tensor, zero_points: torch.Tensor | None,
                   stats: torch.Tensor | None, workspace: torch.Tensor | None, stream=None) -> None:
    """x: bf16 [rows, cols]; col_scale: fp32 [cols] or None; sign_bits: int32 [cols / 32]
    (bit j % 32 of word j / 32 negates column j) or None (no rotation)."""
    rows, cols = x.shape
    sc = scheme.c()
    rt = _rt(col_scale, sign_bits)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib().bq_quantize_rt(_ptr(x), DT["bf16"], rows, cols, ctypes.byref(sc), ctypes.byref(rt), _ptr(codes),
                                 _ptr(scales), _ptr(zero_points), _ptr(stats), _ptr(workspace), ws_bytes,
                                 _stream(stream)), "bq_quantize_rt")


def bq_dequantize_rt(codes: torch.Tensor, scales: torch.Tensor, zero_points: torch.Tensor | None, rows: int,
                     cols: int, scheme: Scheme, col_scale: torch.Tensor | None, sign_bits: torch.Tensor | None,
                     out: torch.Tensor, stream=None) -> None:
    out_dt = {torch.bfloat16: DT["bf16"], torch.float32: DT["fp32"]}[out.dtype]
    sc = scheme.c()
    rt = _rt(col_scale, sign_bits)
    _check(_lib().bq_dequantize_rt(_ptr(codes), _ptr(scales), _ptr(zero_points), rows, cols, ctypes.byref(sc),
                                   ctypes.byref(rt), _ptr(out), out_dt, _stream(stream)), "bq_dequantize_rt")


def pack_sign_bits(signs, device=None) -> torch.Tensor:
    """Per-column 0/1 flags (1 = negate) -> int32 words, bit j % 32 of word j / 32."""
    f = torch.as_tensor(signs).to(torch.int64).reshape(-1, 32)
    w = (f << torch.arange(32, dtype=torch.int64)).sum(1)
    w = torch.where(w >= 2 ** 31, w - 2 ** 32, w).to(torch.int32)
    return w.to(device) if device is not None else w


def bq_wait_timeouts(reset: bool = False) -> int:
    """Tile waits of the quantize kernels that gave up on the current device (each
    leaves its call's outputs incomplete); synchronizes with the device."""
    c = ctypes.c_uint32(0)
    _check(_lib().bq_wait_timeouts(ctypes.byref(c), 1 if reset else 0), "bq_wait_timeouts")
    return int(c.value)


def bq_stats_qsnr_db(stats_host) -> float:
    """QSNR in dB from a host copy of the five stats values (tensor or sequence)."""
    v = [float(a) for a in (stats_host.tolist() if hasattr(stats_host, "tolist") else stats_host)]
    s = BqStats(*v[:5])
    return float(_lib().bq_stats_qsnr_db(ctypes.byref(s)))


def bq_stats_to_db(stats_host) -> float:
    """The same as bq_stats_qsnr_db (the C ABI exports both names)."""
    v = [float(a) for a in (stats_host.tolist() if hasattr(stats_host, "tolist") else stats_host)]
    s = BqStats(*v[:5])
    return float(_lib().bq_stats_to_db(ctypes.byref(s)))


# ---------------------------------------------------------------------------
# Allocation helpers
# ---------------------------------------------------------------------------

def _scale_dtype_torch(scheme: Scheme):
    s = scheme.resolved()
    if s.gran in ("mx", "nv"):
        return torch.uint8
    return torch.float16 if s.scale_dtype == "fp16" else torch.float32


def new_workspace(device=None, nbytes: int | None = None) -> torch.Tensor:
    """A zero-filled workspace large enough for any call (bytes as uint8)."""
    if nbytes is None:
        nbytes = bq_workspace_size(Scheme("int8_sym", "tensor"), 1, 16, True)
    return torch.zeros(nbytes, dtype=torch.uint8, device=device or "cuda")


@dataclass
class Quantized:
    scheme: Scheme
    rows: int
    cols: int
    codes: torch.Tensor
    scales: torch.Tensor
    zero_points: torch.Tensor | None
    tensor_scale: torch.Tensor | None
    stats: torch.Tensor | None      # float64[5] on the device: err2, x2, kappa_sum, kappa_max, n_units

    def qsnr_db(self) -> float:
        return bq_stats_qsnr_db(self.stats.cpu())

    def mean_kappa(self) -> float:
        st = self.stats.cpu().tolist()
        return st[2] / st[4] if st[4] else math.nan


def alloc_outputs(scheme: Scheme, rows: int, cols: int, device, stats: bool = True) -> Quantized:
    s = scheme.resolved()
    cb, sb, zb, tb = bq_buffer_sizes(s, rows, cols)
    sdt = _scale_dtype_torch(s)
    esz = torch.tensor([], dtype=sdt).element_size()
    cols_b = cols // 2 if s.fmt in FOUR_BIT else cols
    codes = torch.empty((rows, cols_b), dtype=torch.uint8, device=device)
    scales = torch.empty(max(sb // esz, 1), dtype=sdt, device=device)
    zps = torch.empty(zb // esz, dtype=sdt, device=device) if zb else None
    ts = torch.empty(1, dtype=torch.float32, device=device) if tb else None
    st = torch.empty(5, dtype=torch.float64, device=device) if stats else None
    return Quantized(s, rows, cols, codes, scales, zps, ts, st)


@dataclass
class QuantizedBatch:
    scheme: Scheme
    batch: int
    rows: int
    cols: int
    codes: torch.Tensor             # uint8 [batch, rows, cols] (4-bit: [batch, rows, cols / 2])
    scales: torch.Tensor            # [batch, one tensor's scales]
    zero_points: torch.Tensor | None
    stats: torch.Tensor | None      # float64 [batch, 5]

    def tensor(self, b: int) -> Quantized:
        """Tensor b's outputs as a Quantized (views, no copy)."""
        return Quantized(self.scheme, self.rows, self.cols, self.codes[b], self.scales[b],
                         None if self.zero_points is None else self.zero_points[b], None,
                         None if self.stats is None else self.stats[b])


def alloc_batch_outputs(scheme: Scheme, batch: int, rows: int, cols: int, device, stats: bool = True) -> QuantizedBatch:
    s = scheme.resolved()
    cb, sb, zb, _ = bq_buffer_sizes(s, rows, cols)
    sdt = _scale_dtype_torch(s)
    esz = torch.tensor([], dtype=sdt).element_size()
    cols_b = cols // 2 if s.fmt in FOUR_BIT else cols
    codes = torch.empty((batch, rows, cols_b), dtype=torch.uint8, device=device)
    scales = torch.empty((batch, max(sb // esz, 1)), dtype=sdt, device=device)
    zps = torch.empty((batch, zb // esz), dtype=sdt, device=device) if zb else None
    st = torch.empty((batch, 5), dtype=torch.float64, device=device) if stats else None
    return QuantizedBatch(s, batch, rows, cols, codes, scales, zps, st)


def quantize_batch(x: torch.Tensor, scheme: Scheme, stats: bool = True, workspace: torch.Tensor | None = None,
                   out: QuantizedBatch | None = None, stream=None) -> QuantizedBatch:
    """Quantize a bf16 [batch, rows, cols] CUDA tensor (same-shape tensors, one launch);
    per-tensor QSNR / kappa sums in stats[b]."""
    if x.dtype != torch.bfloat16 or not x.is_cuda or x.dim() != 3:
        raise ValueError("x must be a 3-D bf16 CUDA tensor")
    x = x.contiguous()
    batch, rows, cols = x.shape
    q = out or alloc_batch_outputs(scheme, batch, rows, cols, x.device, stats)
    if stats and workspace is None:
        workspace = new_workspace(x.device)
    bq_quantize_batch(x, q.scheme, q.codes, q.scales, q.zero_points, q.stats if stats else None, workspace, stream)
    return q


def quantize(x: torch.Tensor, scheme: Scheme, stats: bool = True, workspace: torch.Tensor | None = None,
             out: Quantized | None = None, stream=None) -> Quantized:
    """Quantize a bf16 [rows, cols] CUDA tensor; returns codes, scales, zero points,
    tensor scale and (optionally) the QSNR / kappa sums, all on the device."""
    if x.dtype != torch.bfloat16 or not x.is_cuda or x.dim() != 2:
        raise ValueError("x must be a 2-D bf16 CUDA tensor")
    x = x.contiguous()
    rows, cols = x.shape
    q = out or alloc_outputs(scheme, rows, cols, x.device, stats)
    if workspace is None and bq_workspace_size(q.scheme, rows, cols, stats) > 0:
        workspace = new_workspace(x.device)
    bq_quantize(x, q.scheme, q.codes, q.scales, q.zero_points, q.tensor_scale, q.stats if stats else None,
                workspace, stream)
    return q


def dequantize(q: Quantized, dtype=torch.bfloat16, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty((q.rows, q.cols), dtype=dtype, device=q.codes.device)
    bq_dequantize(q.codes, q.scales, q.zero_points, q.tensor_scale, q.rows, q.cols, q.scheme, out, stream)
    return out


def quantize_rt(x: torch.Tensor, scheme: Scheme, col_scale: torch.Tensor | None = None,
                sign_bits: torch.Tensor | None = None, stats: bool = True, workspace: torch.Tensor | None = None,
                stream=None) -> Quantized:
    """Quantize a bf16 [rows, cols] CUDA tensor after the row transforms (per-column
    factor, randomized full-row Hadamard rotation); per-row, per-group and MX schemes."""
    if x.dtype != torch.bfloat16 or not x.is_cuda or x.dim() != 2:
        raise ValueError("x must be a 2-D bf16 CUDA tensor")
    x = x.contiguous()
    rows, cols = x.shape
    q = alloc_outputs(scheme, rows, cols, x.device, stats)
    if stats and workspace is None:
        workspace = new_workspace(x.device)
    bq_quantize_rt(x, q.scheme, col_scale, sign_bits, q.codes, q.scales, q.zero_points,
                   q.stats if stats else None, workspace, stream)
    return q


def dequantize_rt(q: Quantized, col_scale: torch.Tensor | None = None, sign_bits: torch.Tensor | None = None,
                  dtype=torch.bfloat16, stream=None) -> torch.Tensor:
    out = torch.empty((q.rows, q.cols), dtype=dtype, device=q.codes.device)
    bq_dequantize_rt(q.codes, q.scales, q.zero_points, q.rows, q.cols, q.scheme, col_scale, sign_bits, out, stream)
    return out


def qsnr(x: torch.Tensor, q: Quantized, workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Standalone QSNR sums (float64[5] on the device; kappa fields zero)."""
    st = torch.empty(5, dtype=torch.float64, device=x.device)
    if workspace is None:
        workspace = new_workspace(x.device)
    bq_qsnr(x.contiguous(), q.codes, q.scales, q.zero_points, q.tensor_scale, q.scheme, st, workspace, stream)
    return st
