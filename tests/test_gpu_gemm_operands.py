"""GEMM-ready block scales on the GPU: MX / NV scales written straight into the layout a
block-scaled tensor-core GEMM reads (BQ_LAYOUT_GEMM), checked two ways.

* Parity: codes as in the row-major layout, scale bytes equal to the oracle's scales
  placed by the oracle's layout function, dequantize and QSNR reading the same layout.
* A consumer: the library's block-scaled GEMM (torch's scaled_mm on cuBLASLt, MXFP8
  operands, 1 x 32 UE8M0 blocks, 32x4x4 swizzled scales) fed our codes and scales as
  they are, against the product of the oracle's dequantized operands in float64. A
  wrong scale layout puts scales on the wrong blocks and misses by orders of magnitude.
"""

import numpy as np
import pytest
import torch

import oracle
import synth
import block_scaled_bit_bq_b200 as bq
from block_scaled_bit_bq_b200 import Scheme

pytestmark = pytest.mark.gpu


def _o(s):
    return oracle.Scheme(s.fmt, s.gran, s.block, s.scale_dtype, s.hadamard)


def _nb(s, cols):
    return cols // (32 if s.gran == "mx" else 16)


@pytest.fixture(scope="module")
def ws(cuda_device):
    return bq.new_workspace(cuda_device)


SCHEMES = [Scheme("e4m3", "mx", layout="gemm"), Scheme("e5m2", "mx", layout="gemm"), Scheme("e2m1", "mx", layout="gemm"),
           Scheme("int8_sym", "mx", layout="gemm"), Scheme("e2m3", "mx", layout="gemm"),
           Scheme("e2m1", "nv", layout="gemm"), Scheme("int4_sym", "nv", layout="gemm"),
           Scheme("int4_sym", "nv", hadamard=True, layout="gemm"), Scheme("int8_sym", "mx", hadamard=True, layout="gemm")]


@pytest.mark.parametrize("shape", [(1, 128), (130, 1024), (256, 4096)], ids=lambda t: f"{t[0]}x{t[1]}")
@pytest.mark.parametrize("s", SCHEMES, ids=str)
def test_gemm_layout_parity(s, shape, ws):
    rows, cols = shape
    x = synth.activations_t3(rows, cols, seed=600 + rows, n_outlier_channels=2)
    xb = synth.bf16_bits(x)
    q = bq.quantize(x.cuda(), s, stats=True, workspace=ws)
    d32 = bq.dequantize(q, torch.float32)
    qs = bq.qsnr(x.cuda(), q, workspace=ws)
    torch.cuda.synchronize()
    o = oracle.quantize(xb, _o(s))
    assert np.array_equal(q.codes.cpu().numpy(), o["codes"])
    nb = _nb(s, cols)
    got = q.scales.cpu().numpy().view(np.uint8)
    assert got.size == oracle.gemm_scale_bytes(rows, nb)
    assert np.array_equal(oracle.scales_from_gemm(got, rows, nb), o["scales"].reshape(rows, nb))
    oxh = oracle.dequantize(o["codes"], o["scales"], o["zps"], o["tensor_scale"], rows, cols, _o(s))
    assert np.array_equal(d32.cpu().numpy().view(np.uint32), oxh.view(np.uint32))
    st = q.stats.cpu().numpy()
    assert abs(bq.bq_stats_qsnr_db(st) - oracle.qsnr_db(*o["stats"][:2])) < 0.01
    sums = qs.cpu().numpy()
    assert abs(bq.bq_stats_qsnr_db(sums) - oracle.qsnr_db(*o["stats"][:2])) < 0.01


def test_gemm_layout_with_the_row_rotation(ws):
    rows, cols = 200, 2048
    x = synth.weight_outliers(rows, cols, seed=610)
    sg = synth.random_signs(cols, 611)
    s = Scheme("e2m1", "mx", layout="gemm")
    sb = bq.pack_sign_bits(sg, torch.device("cuda"))
    q = bq.quantize_rt(x.cuda(), s, sign_bits=sb, workspace=ws)
    xh = bq.dequantize_rt(q, None, sb, torch.float32)
    torch.cuda.synchronize()
    o = oracle.quantize_rt(synth.bf16_bits(x), _o(s), signs=sg)
    assert np.array_equal(q.codes.cpu().numpy(), o["codes"])
    got = q.scales.cpu().numpy().view(np.uint8)
    assert np.array_equal(oracle.scales_from_gemm(got, rows, cols // 32), o["scales"].reshape(rows, -1))
    oxh = oracle.dequantize_rt(o["codes"], o["scales"], None, rows, cols, _o(s), signs=sg)
    assert np.array_equal(xh.cpu().numpy().view(np.uint32), oxh.view(np.uint32))


def _scaled_mm_or_skip():
    F = torch.nn.functional
    if not (hasattr(F, "scaled_mm") and hasattr(F, "ScalingType") and hasattr(F, "SwizzleType")
            and hasattr(torch, "float8_e8m0fnu")):
        pytest.skip("this torch has no block-scaled scaled_mm")
    return F


@pytest.mark.parametrize("fmt,tdtype", [("e4m3", "float8_e4m3fn")])     # the library takes no E5M2 x E5M2
def test_block_scaled_gemm_consumes_the_operands(fmt, tdtype, ws):
    F = _scaled_mm_or_skip()
    M, N, K = 256, 384, 2048
    a = synth.activations_t3(M, K, seed=620, n_outlier_channels=4)
    b = synth.weight_outliers(N, K, seed=621)
    s = Scheme(fmt, "mx", layout="gemm")
    qa = bq.quantize(a.cuda(), s, stats=False)
    qb = bq.quantize(b.cuda(), s, stats=False)
    dt = getattr(torch, tdtype)

    def gemm(out_dtype):
        return F.scaled_mm(qa.codes.view(dt), qb.codes.view(dt).t(),
                           qa.scales.view(torch.float8_e8m0fnu), F.ScalingType.BlockWise1x32,
                           qb.scales.view(torch.float8_e8m0fnu), F.ScalingType.BlockWise1x32,
                           swizzle_a=F.SwizzleType.SWIZZLE_32_4_4, swizzle_b=F.SwizzleType.SWIZZLE_32_4_4,
                           output_dtype=out_dtype)

    out_rel = 0.0                      # the output's own rounding
    try:
        c = gemm(torch.float32)
    except RuntimeError:
        try:
            c = gemm(torch.bfloat16)
            out_rel = 2.0 ** -8
        except RuntimeError as e:
            pytest.skip(f"the library GEMM does not take these operands: {e}")
    torch.cuda.synchronize()
    os_ = _o(s)
    oa = oracle.quantize(synth.bf16_bits(a), os_, stats=False)
    ob = oracle.quantize(synth.bf16_bits(b), os_, stats=False)
    da = oracle.dequantize(oa["codes"], oa["scales"], None, None, M, K, os_).astype(np.float64)
    db = oracle.dequantize(ob["codes"], ob["scales"], None, None, N, K, os_).astype(np.float64)
    ref = da @ db.T
    mag = np.abs(da) @ np.abs(db).T
    got = c.cpu().numpy().astype(np.float64)
    # fp32 accumulation of exact products: well inside 1e-4 of the sum of |products|
    assert np.all(np.abs(got - ref) <= 1e-4 * mag + out_rel * np.abs(ref) + 1e-30)
    assert np.max(np.abs(ref)) > 0
