"""Host-side checks of the C ABI (no GPU, no compute calls).

libbq.so loads, exports every function include/bq.h declares, sizes buffers the way
the oracle does, and rejects bad schemes, shapes, pointers, alignment and workspaces
on the host before any launch.
"""

import ctypes
import os
import re

import pytest

import oracle
import block_scaled_bit_bq_b200 as bq
from block_scaled_bit_bq_b200 import Scheme

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "bq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\*?\s+\**(bq_[a-z_0-9]+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_library_exports_every_declared_function():
    names = _declared_functions()
    assert {"bq_quantize", "bq_dequantize", "bq_qsnr", "bq_buffer_sizes", "bq_workspace_size",
            "bq_stats_qsnr_db", "bq_status_string", "bq_version"} <= set(names)
    L = ctypes.CDLL(bq.LIB_PATH)
    for n in names:
        assert hasattr(L, n), n
    assert "sm_100a" in bq.bq_version()


SCHEMES = [
    Scheme("int8_sym", "tensor"), Scheme("int8_sym", "row"), Scheme("int8_sym", "group", 64),
    Scheme("int8_asym", "tensor"), Scheme("int8_asym", "row", scale_dtype="fp16"),
    Scheme("int8_asym", "group", 128, "fp16"), Scheme("int4_sym", "group", 64),
    Scheme("uint4_asym", "group", 128, "fp16"), Scheme("e4m3", "tensor"), Scheme("e5m2", "row"),
    Scheme("int8_sym", "mx"), Scheme("e4m3", "mx"), Scheme("e5m2", "mx"), Scheme("e2m1", "mx"),
    Scheme("e2m3", "mx"), Scheme("e3m2", "mx"),
    Scheme("e2m1", "nv"), Scheme("int4_sym", "nv"), Scheme("int4_sym", "nv", hadamard=True),
    Scheme("int8_sym", "group", 512), Scheme("e4m3", "group", 16, "fp16"),
    Scheme("e4m3", "tile2d"), Scheme("uint4_asym", "tile2d", scale_dtype="fp16"), Scheme("int4_sym", "tile2d"),
]

GEMM_SCHEMES = [Scheme("e4m3", "mx", layout="gemm"), Scheme("e2m1", "mx", layout="gemm"),
                Scheme("e2m1", "nv", layout="gemm"), Scheme("int8_sym", "mx", layout="gemm")]


@pytest.mark.parametrize("s", GEMM_SCHEMES, ids=str)
@pytest.mark.parametrize("shape", [(1, 128), (130, 1024), (4096, 4096)])
def test_gemm_layout_buffer_sizes(s, shape):
    rows, cols = shape
    o = oracle.Scheme(s.fmt, s.gran, s.block, s.scale_dtype, s.hadamard)
    cb, sb, zb, tb = oracle.buffer_sizes(o, rows, cols)
    nb = cols // (32 if s.gran == "mx" else 16)
    assert bq.bq_buffer_sizes(s, rows, cols) == (cb, oracle.gemm_scale_bytes(rows, nb), zb, tb)


@pytest.mark.parametrize("s", SCHEMES, ids=str)
@pytest.mark.parametrize("shape", [(1, 512), (37, 1024), (4096, 4096), (0, 512)])
def test_buffer_sizes_match_oracle(s, shape):
    rows, cols = shape
    o = oracle.Scheme(s.fmt, s.gran, s.block, s.scale_dtype, s.hadamard)
    assert bq.bq_buffer_sizes(s, rows, cols) == oracle.buffer_sizes(o, rows, cols)


def test_workspace_only_when_needed():
    assert bq.bq_workspace_size(Scheme("int8_sym", "row"), 8, 64, False) == 0
    assert bq.bq_workspace_size(Scheme("int4_sym", "group", 64), 8, 64, False) == 0
    assert bq.bq_workspace_size(Scheme("int8_sym", "row"), 8, 64, True) > 0
    assert bq.bq_workspace_size(Scheme("e4m3", "tensor"), 8, 64, False) > 0
    assert bq.bq_workspace_size(Scheme("e2m1", "nv"), 8, 64, False) > 0


def _status(fn, *args):
    try:
        fn(*args)
    except bq.BqError as e:
        return e.status
    return 0


@pytest.mark.parametrize("s,shape,want", [
    (Scheme("e2m1", "row"), (4, 64), 2),
    (Scheme("e2m1", "tensor"), (4, 64), 2),
    (Scheme("e2m3", "row"), (4, 64), 2),
    (Scheme("e3m2", "group", 32), (4, 64), 2),
    (Scheme("e3m2", "nv"), (4, 64), 2),
    (Scheme("int8_asym", "mx"), (4, 64), 2),
    (Scheme("e4m3", "nv"), (4, 64), 2),
    (Scheme("int8_sym", "group", 48), (4, 96), 2),
    (Scheme("int8_sym", "mx", 16), (4, 64), 2),
    (Scheme("int8_sym", "row", scale_dtype="e4m3"), (4, 64), 2),
    (Scheme("int8_sym", "row"), (4, 24), 3),
    (Scheme("int8_sym", "row"), (-1, 64), 3),
    (Scheme("int8_sym", "group", 128), (4, 64), 3),
    (Scheme("int8_sym", "row"), (1 << 20, 1 << 16), 3),      # 2^36 elements
    (Scheme("int8_sym", "row"), (4, 0), 3),
    (Scheme("e2m1", "tile2d"), (4, 128), 2),
    (Scheme("e2m3", "tile2d"), (4, 128), 2),
    (Scheme("int8_sym", "tile2d", 64), (4, 128), 2),
    (Scheme("int8_sym", "tile2d", scale_dtype="ue8m0"), (4, 128), 2),
    (Scheme("int8_sym", "tile2d"), (4, 192), 3),
    (Scheme("int8_sym", "row", layout="gemm"), (4, 128), 2),
    (Scheme("e4m3", "group", 32, layout="gemm"), (4, 128), 2),
    (Scheme("e4m3", "mx", layout="gemm"), (4, 96), 3),
    (Scheme("e2m1", "nv", layout="gemm"), (4, 112), 3),
    # one row of 2^31 - 128 columns: 2^36 padded scale bytes, past 32-bit offsets
    (Scheme("e2m1", "nv", layout="gemm"), (1, (1 << 31) - 128), 3),
])
def test_invalid_schemes_and_shapes(s, shape, want):
    assert _status(bq.bq_buffer_sizes, s, *shape) == want


def test_bad_enum_and_reserved():
    L = bq.lib()
    z = ctypes.c_size_t(0)
    for f in [(9, 0, 0, 2, 0, 0), (0, 7, 0, 2, 0, 0), (0, 6, 0, 2, 0, 0), (0, 1, 0, 2, 2, 0), (0, 1, 0, 2, 0, 2), (0, 1, 0, 9, 0, 0)]:
        sc = bq.BqScheme(*f)
        assert L.bq_buffer_sizes(ctypes.byref(sc), 4, 64, ctypes.byref(z), None, None, None) == 1
    assert L.bq_buffer_sizes(None, 4, 64, ctypes.byref(z), None, None, None) == 1


def test_quantize_argument_checks_happen_before_any_launch():
    L = bq.lib()
    sc = Scheme("int8_sym", "row").c()
    nv = Scheme("e2m1", "nv").c()
    asym = Scheme("uint4_asym", "group", 128, "fp16").c()
    fake = 1 << 40        # never dereferenced: every call below fails its host checks
    ws = ctypes.c_void_p(fake)
    # null x / codes / scales
    assert L.bq_quantize(None, 0, 4, 64, ctypes.byref(sc), fake, fake, None, None, None, None, 0, None) == 1
    assert L.bq_quantize(fake, 0, 4, 64, ctypes.byref(sc), None, fake, None, None, None, None, 0, None) == 1
    # asymmetric without zero points; NV without tensor scale
    assert L.bq_quantize(fake, 0, 4, 128, ctypes.byref(asym), fake, fake, None, None, None, None, 0, None) == 1
    assert L.bq_quantize(fake, 0, 4, 64, ctypes.byref(nv), fake, fake, None, None, None, ws, 1 << 20, None) == 1
    # misaligned x or codes
    assert L.bq_quantize(fake + 16, 0, 4, 64, ctypes.byref(sc), fake, fake, None, None, None, None, 0, None) == 4
    assert L.bq_quantize(fake, 0, 4, 64, ctypes.byref(sc), fake + 8, fake, None, None, None, None, 0, None) == 4
    # stats without a workspace; NV without a workspace; a workspace too small
    assert L.bq_quantize(fake, 0, 4, 64, ctypes.byref(sc), fake, fake, None, None, fake, None, 0, None) == 5
    assert L.bq_quantize(fake, 0, 4, 64, ctypes.byref(nv), fake, fake, None, fake, None, None, 0, None) == 5
    assert L.bq_quantize(fake, 0, 4, 64, ctypes.byref(sc), fake, fake, None, None, fake, ws, 64, None) == 5
    # unsupported input dtype
    assert L.bq_quantize(fake, 2, 4, 64, ctypes.byref(sc), fake, fake, None, None, None, None, 0, None) == 2
    # dequantize: bad output dtype, misaligned output, missing pointers
    assert L.bq_dequantize(fake, fake, None, None, 4, 64, ctypes.byref(sc), fake, 1, None) == 2
    assert L.bq_dequantize(fake, fake, None, None, 4, 64, ctypes.byref(sc), fake + 4, 0, None) == 4
    assert L.bq_dequantize(None, fake, None, None, 4, 64, ctypes.byref(sc), fake, 0, None) == 1
    # qsnr: stats and workspace are required
    assert L.bq_qsnr(fake, 0, fake, fake, None, None, 4, 64, ctypes.byref(sc), None, ws, 1 << 20, None) == 1
    assert L.bq_qsnr(fake, 0, fake, fake, None, None, 4, 64, ctypes.byref(sc), fake, None, 0, None) == 5


def test_empty_dequantize_is_a_no_op():
    L = bq.lib()
    sc = Scheme("int8_sym", "row").c()
    assert L.bq_dequantize(None, None, None, None, 0, 64, ctypes.byref(sc), None, 0, None) == 0


def test_stats_to_db():
    # -10 log10(0.0234375 / 2.9453125) = 20.99219 dB
    for f in (bq.bq_stats_qsnr_db, bq.bq_stats_to_db):
        assert abs(f([0.0234375, 2.9453125, 0, 0, 0]) - 20.99219) < 1e-4
        assert f([0.0, 1.0, 0, 0, 0]) == float("inf")
    # the C symbol bq_stats_to_db itself, through ctypes
    L = bq.lib()
    s = bq.BqStats(1.0, 1000.0, 0.0, 0.0, 0.0)
    assert abs(L.bq_stats_to_db(ctypes.byref(s)) - 30.0) < 1e-12
    assert L.bq_stats_to_db(None) != L.bq_stats_to_db(None)        # NaN for a NULL pointer


def test_range_split_checks_before_any_launch():
    L = bq.lib()
    fake = 1 << 40
    ws = ctypes.c_void_p(fake)
    t = Scheme("e4m3", "tensor").c()
    row = Scheme("int8_sym", "row").c()
    # only per-tensor and NV schemes have a range pass
    assert L.bq_tensor_range(fake, 0, 4, 64, ctypes.byref(row), fake, ws, 1 << 20, None) == 2
    assert L.bq_quantize_with_range(fake, 0, 4, 64, ctypes.byref(row), fake, fake, fake, None, None, None,
                                    None, 0, None) == 2
    # range output / input required; workspace required for the range pass
    assert L.bq_tensor_range(fake, 0, 4, 64, ctypes.byref(t), None, ws, 1 << 20, None) == 1
    assert L.bq_tensor_range(fake, 0, 4, 64, ctypes.byref(t), fake, None, 0, None) == 5
    assert L.bq_quantize_with_range(fake, 0, 4, 64, ctypes.byref(t), None, fake, fake, None, None, None,
                                    None, 0, None) == 1
    # alignment: x 32 bytes, the range 4 bytes
    assert L.bq_tensor_range(fake + 16, 0, 4, 64, ctypes.byref(t), fake, ws, 1 << 20, None) == 4
    assert L.bq_tensor_range(fake, 0, 4, 64, ctypes.byref(t), fake + 2, ws, 1 << 20, None) == 4
    assert L.bq_quantize_with_range(fake, 0, 4, 64, ctypes.byref(t), fake + 1, fake, fake, None, None, None,
                                    None, 0, None) == 4
    # stats need a workspace; an NV scheme needs its tensor scale output
    assert L.bq_quantize_with_range(fake, 0, 4, 64, ctypes.byref(t), fake, fake, fake, None, None, fake,
                                    None, 0, None) == 5
    nv = Scheme("e2m1", "nv").c()
    assert L.bq_quantize_with_range(fake, 0, 4, 64, ctypes.byref(nv), fake, fake, fake, None, None, None,
                                    None, 0, None) == 1


def test_batch_checks_before_any_launch():
    L = bq.lib()
    fake = 1 << 40
    ws = ctypes.c_void_p(fake)
    mx = Scheme("int8_sym", "mx").c()
    def q(scheme, batch, rows, cols, x=fake, codes=fake, stats=None, wsb=0):
        return L.bq_quantize_batch(x, 0, batch, rows, cols, ctypes.byref(scheme), codes, fake, None, stats,
                                   ws if wsb else None, wsb, None)
    # per-tensor, NV and 2-D tile schemes, and per-row widths off the flat kernel, are not offered
    for s, cols in [(Scheme("e4m3", "tensor"), 64), (Scheme("e2m1", "nv"), 64), (Scheme("e4m3", "tile2d"), 128),
                    (Scheme("int8_sym", "row"), 4096), (Scheme("int8_sym", "row"), 192)]:
        assert q(s.c(), 2, 4, cols) == 2
    assert q(mx, -1, 4, 64) == 3                                 # negative batch
    assert q(mx, 2, 1, 32) == 3                                  # tensors of a partial 64-element span
    assert q(Scheme("e4m3", "mx", layout="gemm").c(), 2, 64, 128) == 3    # GEMM layout: rows % 128
    assert q(mx, 2, 4, 64, x=None) == 1
    assert q(mx, 2, 4, 64, x=fake + 16) == 4
    assert q(mx, 2, 4, 64, stats=fake) == 5                      # stats without a workspace
    assert q(mx, 0, 4, 64, x=None, codes=None) == 0              # an empty batch is a no-op


def test_debug_hook_rejects_negative_tiles():
    assert bq.lib().bq_debug_skip_tile_copy(-1) == 1


def test_status_strings():
    for k in range(7):
        assert bq.bq_status_string(k).startswith(bq.STATUS[k])


def test_row_transform_checks_before_any_launch():
    L = bq.lib()
    fake = 1 << 40
    ws = ctypes.c_void_p(fake)
    row = Scheme("int8_sym", "row").c()
    rt_rot = bq.BqRowTransform(None, fake, 0)
    def q(scheme, cols, rt, x=fake):
        return L.bq_quantize_rt(x, 0, 4, cols, ctypes.byref(scheme), rt and ctypes.byref(rt), fake, fake, fake,
                                None, None, 0, None)
    # tensor / NV / tile granularities and the block-16 Hadamard are not offered
    for s in [Scheme("int8_sym", "tensor"), Scheme("e2m1", "nv"), Scheme("e4m3", "tile2d"),
              Scheme("int8_sym", "row", hadamard=True)]:
        assert q(s.c(), 512, rt_rot) == 2
    # widths: a multiple of 512 up to 16384, a power of two when rotating
    assert q(row, 256, rt_rot) == 3
    assert q(row, 32768, rt_rot) == 3
    assert q(row, 1536, rt_rot) == 3
    # misaligned factor array, misaligned x, reserved field
    assert q(row, 512, bq.BqRowTransform(fake + 4, None, 0)) == 4
    assert q(row, 512, rt_rot, x=fake + 16) == 4
    assert q(row, 512, bq.BqRowTransform(None, fake, 1)) == 1
    # stats without a workspace
    assert L.bq_quantize_rt(fake, 0, 4, 512, ctypes.byref(row), ctypes.byref(rt_rot), fake, fake, None,
                            fake, None, 0, None) == 5
    assert L.bq_dequantize_rt(fake, fake, None, 4, 1536, ctypes.byref(row), ctypes.byref(rt_rot), fake, 0, None) == 3
