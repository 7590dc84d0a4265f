"""CPU oracle for block-scaled tensor quantization (ctypes front end of bq_oracle.c).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` use it. The CUDA library never imports, links or calls it, and it
shares no code with that library.

The arithmetic lives in ``bq_oracle.c`` (plain C loops, no SIMD, ``-ffp-contract=off``,
no fast-math), which cites the pages each step follows. This module only builds the
shared library, marshals numpy arrays, and names schemes by string:

  fmt:         int8_sym | int8_asym | int4_sym | uint4_asym | e4m3 | e5m2 | e2m1 | e2m3 | e3m2
               (e2m3, e3m2: FP6, MX granularity only, one code per byte)
  gran:        tensor | row | group | mx | nv | tile2d (one scale per 128 x 128 tile)
  scale_dtype: fp32 | fp16 | ue8m0 | e4m3   (default: ue8m0 for mx, e4m3 for nv, else fp32)
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bq_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

FMTS = {"int8_sym": 0, "int8_asym": 1, "int4_sym": 2, "uint4_asym": 3,
        "e4m3": 4, "e5m2": 5, "e2m1": 6, "e2m3": 7, "e3m2": 8}
GRANS = {"tensor": 0, "row": 1, "group": 2, "mx": 3, "nv": 4, "tile2d": 5}
SDTS = {"fp32": 0, "fp16": 1, "ue8m0": 2, "e4m3": 3}
FOUR_BIT = {"int4_sym", "uint4_asym", "e2m1"}
ASYM = {"int8_asym", "uint4_asym"}

CFLAGS = ["-O2", "-std=gnu11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]


def build(force: bool = False) -> str:
    """Compile bq_oracle.c into liboracle.so next to it (if missing or stale)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"], check=True)
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        i64, i32, vp, f32, f64 = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_float, ctypes.c_double
        L.orc_fp_decode.restype = f64
        L.orc_fp_decode.argtypes = [i32, ctypes.c_uint]
        L.orc_fp_encode.restype = ctypes.c_uint
        L.orc_fp_encode.argtypes = [i32, f32]
        L.orc_bf16_to_f32.restype = f32
        L.orc_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.orc_f32_to_bf16.restype = ctypes.c_uint16
        L.orc_f32_to_bf16.argtypes = [f32]
        L.orc_f32_to_f16.restype = ctypes.c_uint16
        L.orc_f32_to_f16.argtypes = [f32]
        L.orc_f16_to_f32.restype = f32
        L.orc_f16_to_f32.argtypes = [ctypes.c_uint16]
        L.orc_ue8m0_exponent.restype = i32
        L.orc_ue8m0_exponent.argtypes = [f32, f32]
        L.orc_fwht16.restype = None
        L.orc_fwht16.argtypes = [vp]
        L.orc_tensor_range.restype = i32
        L.orc_tensor_range.argtypes = [vp, i64, i64, i32, vp]
        L.orc_quantize.restype = i32
        L.orc_quantize.argtypes = [vp, i64, i64, i32, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp]
        L.orc_dequantize.restype = i32
        L.orc_dequantize.argtypes = [vp, vp, vp, vp, i64, i64, i32, i32, i32, i32, i32, vp]
        L.orc_qsnr_sums.restype = i32
        L.orc_qsnr_sums.argtypes = [vp, vp, vp, vp, vp, i64, i64, i32, i32, i32, i32, i32, vp]
        L.orc_qsnr_db.restype = f64
        L.orc_qsnr_db.argtypes = [f64, f64]
        L.orc_f32_to_bf16_array.restype = None
        L.orc_f32_to_bf16_array.argtypes = [vp, vp, i64]
        L.orc_buffer_sizes.restype = i32
        L.orc_buffer_sizes.argtypes = [i32, i32, i32, i32, i32, i64, i64, vp]
        L.orc_fwht.restype = None
        L.orc_fwht.argtypes = [vp, i64]
        L.orc_rotate_rows.restype = i32
        L.orc_rotate_rows.argtypes = [vp, i64, i64, vp, vp, vp]
        L.orc_quantize_rt.restype = i32
        L.orc_quantize_rt.argtypes = [vp, i64, i64, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp]
        L.orc_dequantize_rt.restype = i32
        L.orc_dequantize_rt.argtypes = [vp, vp, vp, i64, i64, i32, i32, i32, i32, vp, vp]
        L.orc_gemm_scale_offset.restype = i64
        L.orc_gemm_scale_offset.argtypes = [i64, i64, i64]
        L.orc_gemm_scale_bytes.restype = i64
        L.orc_gemm_scale_bytes.argtypes = [i64, i64]
        L.orc_scales_to_gemm.restype = None
        L.orc_scales_to_gemm.argtypes = [vp, i64, i64, vp]
        L.orc_scales_from_gemm.restype = None
        L.orc_scales_from_gemm.argtypes = [vp, i64, i64, vp]
        _lib = L
    return _lib


@dataclass(frozen=True)
class Scheme:
    fmt: str
    gran: str
    block: int = 0
    scale_dtype: str | None = None
    hadamard: bool = False

    def resolved(self) -> "Scheme":
        sd = self.scale_dtype
        if sd is None:
            sd = {"mx": "ue8m0", "nv": "e4m3"}.get(self.gran, "fp32")
        blk = self.block
        if blk == 0:
            blk = {"mx": 32, "nv": 16, "tile2d": 128}.get(self.gran, 0)
        return Scheme(self.fmt, self.gran, blk, sd, bool(self.hadamard))

    def args(self):
        s = self.resolved()
        return (FMTS[s.fmt], GRANS[s.gran], int(s.block), SDTS[s.scale_dtype], int(s.hadamard))


def _ptr(a) -> int | None:
    return None if a is None else a.ctypes.data


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what}: invalid scheme or shape (code {rc})")


def buffer_sizes(scheme: Scheme, rows: int, cols: int):
    out = np.zeros(4, dtype=np.int64)
    _check(lib().orc_buffer_sizes(*scheme.args(), rows, cols, _ptr(out)), "buffer_sizes")
    return tuple(int(v) for v in out)


def _scale_np_dtype(scheme: Scheme):
    s = scheme.resolved()
    if s.gran in ("mx", "nv"):
        return np.uint8
    return np.uint16 if s.scale_dtype == "fp16" else np.float32


def quantize(x_bits: np.ndarray, scheme: Scheme, tensor_range=None, stats: bool = True):
    """Quantize a bf16 matrix given as uint16 bits [rows, cols].

    Returns a dict with ``codes`` (uint8), ``scales`` (float32, uint16 fp16 bits, or
    uint8 codes), ``zps`` (same dtype as scales, asymmetric formats only),
    ``tensor_scale`` (float32[1], nv only) and ``stats`` (float64[5]: err2, x2,
    kappa sum, kappa max, units) when requested.
    """
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    rows, cols = x_bits.shape
    s = scheme.resolved()
    cb, sb, zb, tb = buffer_sizes(s, rows, cols)
    sdt = _scale_np_dtype(s)
    codes = np.zeros(cb, dtype=np.uint8)
    scales = np.zeros(sb // np.dtype(sdt).itemsize, dtype=sdt)
    zps = np.zeros(zb // np.dtype(sdt).itemsize, dtype=sdt) if zb else None
    ts = np.zeros(1, dtype=np.float32) if tb else None
    st = np.zeros(5, dtype=np.float64) if stats else None
    tr = None if tensor_range is None else np.asarray(tensor_range, dtype=np.float32)
    rc = lib().orc_quantize(_ptr(x_bits), rows, cols, *s.args(), _ptr(tr), _ptr(codes),
                            _ptr(scales), _ptr(zps), _ptr(ts), _ptr(st))
    _check(rc, "quantize")
    cols_b = cols // 2 if s.fmt in FOUR_BIT else cols
    out = {"codes": codes.reshape(rows, cols_b), "scales": scales, "zps": zps,
           "tensor_scale": ts, "stats": st}
    return out


def dequantize(codes, scales, zps, tensor_scale, rows: int, cols: int, scheme: Scheme) -> np.ndarray:
    """fp32 [rows, cols] dequantized values (inverse rotation applied if set)."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.zeros((rows, cols), dtype=np.float32)
    ts = None if tensor_scale is None else np.ascontiguousarray(tensor_scale, dtype=np.float32)
    rc = lib().orc_dequantize(_ptr(codes), _ptr(np.ascontiguousarray(scales)),
                              _ptr(None if zps is None else np.ascontiguousarray(zps)),
                              _ptr(ts), rows, cols, *scheme.args(), _ptr(out))
    _check(rc, "dequantize")
    return out


def qsnr_sums(x_bits, codes, scales, zps, tensor_scale, scheme: Scheme) -> np.ndarray:
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    rows, cols = x_bits.shape
    st = np.zeros(5, dtype=np.float64)
    ts = None if tensor_scale is None else np.ascontiguousarray(tensor_scale, dtype=np.float32)
    rc = lib().orc_qsnr_sums(_ptr(x_bits), _ptr(np.ascontiguousarray(codes, dtype=np.uint8)),
                             _ptr(np.ascontiguousarray(scales)),
                             _ptr(None if zps is None else np.ascontiguousarray(zps)),
                             _ptr(ts), rows, cols, *scheme.args(), _ptr(st))
    _check(rc, "qsnr_sums")
    return st


def gemm(a: dict, b: dict, m: int, n: int, k: int, scheme: Scheme) -> np.ndarray:
    """D[m, n] = sum_k A[m, k] B[n, k] in float64 of the two operands as quantized (the
    oracle's own quantize outputs a and b, row-layout scales): each operand dequantized
    by the oracle (fp32 values, NV tensor scale and inverse rotation included), then one
    float64 matrix product. This is the block-scaled GEMM's definition: "Quantization
    survey" §4.3.2 (x = x_q s_block S_tensor) and the FP8 recipe's fp8_matmul, whose
    result the tensor cores approximate with fp32 accumulation. A weight W[out, in] is B
    (n = out), so D = A W^T."""
    da = dequantize(a["codes"], a["scales"], a["zps"], a["tensor_scale"], m, k, scheme).astype(np.float64)
    db = dequantize(b["codes"], b["scales"], b["zps"], b["tensor_scale"], n, k, scheme).astype(np.float64)
    return da @ db.T


def gemm_magnitude(a: dict, b: dict, m: int, n: int, k: int, scheme: Scheme) -> np.ndarray:
    """sum_k |A[m, k]| |B[n, k]| of the dequantized operands (the scale of the rounding
    error of any order of summation)."""
    da = np.abs(dequantize(a["codes"], a["scales"], a["zps"], a["tensor_scale"], m, k, scheme).astype(np.float64))
    db = np.abs(dequantize(b["codes"], b["scales"], b["zps"], b["tensor_scale"], n, k, scheme).astype(np.float64))
    return da @ db.T


def tensor_range(x_bits: np.ndarray, hadamard: bool = False):
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    rows, cols = x_bits.shape
    out = np.zeros(3, dtype=np.float32)
    _check(lib().orc_tensor_range(_ptr(x_bits), rows, cols, int(hadamard), _ptr(out)), "tensor_range")
    return out


def qsnr_db(err2: float, x2: float) -> float:
    return float(lib().orc_qsnr_db(float(err2), float(x2)))


def fp_decode(fmt: str, code: int) -> float:
    return float(lib().orc_fp_decode(FMTS[fmt], int(code)))


def fp_encode(fmt: str, v: float) -> int:
    return int(lib().orc_fp_encode(FMTS[fmt], float(v)))


def bf16_to_f32(bits: int) -> float:
    return float(lib().orc_bf16_to_f32(int(bits)))


def f32_to_bf16(v: float) -> int:
    return int(lib().orc_f32_to_bf16(float(v)))


def f32_to_f16(v: float) -> int:
    return int(lib().orc_f32_to_f16(float(v)))


def f16_to_f32(bits: int) -> float:
    return float(lib().orc_f16_to_f32(int(bits)))


def ue8m0_exponent(amax: float, qmax: float) -> int:
    return int(lib().orc_ue8m0_exponent(float(amax), float(qmax)))


def fwht16(v) -> np.ndarray:
    y = np.ascontiguousarray(np.asarray(v, dtype=np.float32).copy())
    assert y.shape == (16,)
    lib().orc_fwht16(_ptr(y))
    return y


def to_bf16_array(values_f32: np.ndarray) -> np.ndarray:
    """fp32 array -> bf16 bits (uint16) with the oracle's own RNE rounding."""
    a = np.ascontiguousarray(values_f32, dtype=np.float32)
    out = np.zeros(a.shape, dtype=np.uint16)
    lib().orc_f32_to_bf16_array(_ptr(a), _ptr(out), a.size)
    return out


# ---------------------------------------------------------------------------
# Row transforms: a per-column factor (SmoothQuant) and the randomized full-row
# Hadamard rotation (QuaRot); signs are bytes, nonzero = -1.
# ---------------------------------------------------------------------------

def _opt_f32(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float32)


def _opt_u8(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.uint8)


def fwht(v: np.ndarray) -> np.ndarray:
    """Unnormalised Walsh-Hadamard transform (Sylvester order) of a float32 vector."""
    v = np.array(v, dtype=np.float32)
    lib().orc_fwht(_ptr(v), v.size)
    return v


def rotate_rows(x_bits: np.ndarray, col_scale=None, signs=None) -> np.ndarray:
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    rows, cols = x_bits.shape
    out = np.zeros((rows, cols), dtype=np.float32)
    cs, sg = _opt_f32(col_scale), _opt_u8(signs)
    _check(lib().orc_rotate_rows(_ptr(x_bits), rows, cols, _ptr(cs), _ptr(sg), _ptr(out)), "rotate_rows")
    return out


def quantize_rt(x_bits: np.ndarray, scheme: Scheme, col_scale=None, signs=None, stats: bool = True):
    """quantize() after the row transforms (row, group and MX schemes)."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    rows, cols = x_bits.shape
    s = scheme.resolved()
    if s.hadamard:
        raise ValueError("oracle quantize_rt: the block-16 Hadamard does not combine with the row transforms")
    cb, sb, zb, tb = buffer_sizes(s, rows, cols)
    sdt = _scale_np_dtype(s)
    codes = np.zeros(cb, dtype=np.uint8)
    scales = np.zeros(sb // np.dtype(sdt).itemsize, dtype=sdt)
    zps = np.zeros(zb // np.dtype(sdt).itemsize, dtype=sdt) if zb else None
    st = np.zeros(5, dtype=np.float64) if stats else None
    cs, sg = _opt_f32(col_scale), _opt_u8(signs)
    a = s.args()
    rc = lib().orc_quantize_rt(_ptr(x_bits), rows, cols, a[0], a[1], a[2], a[3], _ptr(cs), _ptr(sg),
                               _ptr(codes), _ptr(scales), _ptr(zps), _ptr(st))
    _check(rc, "quantize_rt")
    cols_b = cols // 2 if s.fmt in FOUR_BIT else cols
    return {"codes": codes.reshape(rows, cols_b), "scales": scales, "zps": zps, "tensor_scale": None, "stats": st}


def dequantize_rt(codes, scales, zps, rows: int, cols: int, scheme: Scheme, signs=None) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.zeros((rows, cols), dtype=np.float32)
    sg = _opt_u8(signs)
    a = scheme.resolved().args()
    rc = lib().orc_dequantize_rt(_ptr(codes), _ptr(np.ascontiguousarray(scales)),
                                 _ptr(None if zps is None else np.ascontiguousarray(zps)), rows, cols,
                                 a[0], a[1], a[2], a[3], _ptr(sg), _ptr(out))
    _check(rc, "dequantize_rt")
    return out


# ---------------------------------------------------------------------------
# MX / NV block scales in a block-scaled GEMM's layout (128 x 4 tiles of 512 bytes)
# ---------------------------------------------------------------------------

def gemm_scale_bytes(rows: int, nb: int) -> int:
    return int(lib().orc_gemm_scale_bytes(rows, nb))


def gemm_scale_offset(r: int, c: int, nb: int) -> int:
    return int(lib().orc_gemm_scale_offset(r, c, nb))


def scales_to_gemm(scales: np.ndarray, rows: int, nb: int, fill: int = 0) -> np.ndarray:
    """Row-major [rows, nb] uint8 scale codes -> the GEMM layout (padding = fill)."""
    a = np.ascontiguousarray(scales, dtype=np.uint8).reshape(rows, nb)
    out = np.full(gemm_scale_bytes(rows, nb), fill, dtype=np.uint8)
    lib().orc_scales_to_gemm(_ptr(a), rows, nb, _ptr(out))
    return out


def scales_from_gemm(buf: np.ndarray, rows: int, nb: int) -> np.ndarray:
    b = np.ascontiguousarray(buf, dtype=np.uint8)
    out = np.zeros((rows, nb), dtype=np.uint8)
    lib().orc_scales_from_gemm(_ptr(b), rows, nb, _ptr(out))
    return out
