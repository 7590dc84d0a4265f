"""The block-scaled GEMM on the tensor cores (bq_gemm) against the oracle.

A and B are quantized on the GPU into GEMM-layout scales (their codes and scales equal
the oracle's, checked again here); bq_gemm's D is compared with oracle.gemm, the float64
product of the oracle's dequantized operands. Every product of codes and scales is exact,
so the only error is the fp32 accumulation on the tensor cores. Its typical size is
about sqrt(K) 2^-24 of sum |a||b| (4e-6 at K = 4096), well inside the 1e-4 of sum |a||b|
allowed here, while a block scale on the wrong block, a transposed operand or a lost
tensor scale misses by orders of magnitude.
"""

import numpy as np
import pytest
import torch

import oracle
import synth
import block_scaled_bit_bq_b200 as bq
from block_scaled_bit_bq_b200 import Scheme

pytestmark = pytest.mark.gpu

REL = 1e-4


def _o(s):
    return oracle.Scheme(s.fmt, s.gran, s.block, s.scale_dtype, s.hadamard)


def _operands(s, m, n, k, seed):
    a = synth.activations_t3(m, k, seed=seed, n_outlier_channels=3)
    b = synth.weight_outliers(n, k, seed=seed + 1)
    return a, b


def _run(s, m, n, k, seed, dtype=torch.float32):
    a, b = _operands(s, m, n, k, seed)
    qa = bq.quantize(a.cuda(), s, stats=False)
    qb = bq.quantize(b.cuda(), s, stats=False)
    d = bq.gemm(qa, qb, dtype)
    torch.cuda.synchronize()
    os_ = _o(s)
    oa = oracle.quantize(synth.bf16_bits(a), os_, stats=False)
    ob = oracle.quantize(synth.bf16_bits(b), os_, stats=False)
    assert np.array_equal(qa.codes.cpu().numpy(), oa["codes"]) and np.array_equal(qb.codes.cpu().numpy(), ob["codes"])
    ref = oracle.gemm(oa, ob, m, n, k, os_)
    mag = oracle.gemm_magnitude(oa, ob, m, n, k, os_)
    got = d.float().cpu().numpy().astype(np.float64)
    out_rel = 2.0 ** -8 if dtype == torch.bfloat16 else 0.0
    bad = np.abs(got - ref) > REL * mag + out_rel * np.abs(ref) + 1e-30
    assert not bad.any(), (s, (m, n, k), np.argwhere(bad)[:5], got[bad][:5], ref[bad][:5])
    assert np.max(np.abs(ref)) > 0
    return got, ref


MX = Scheme("e4m3", "mx", layout="gemm")
NV = Scheme("e2m1", "nv", layout="gemm")


# one CTA and one k-stage first: the smallest case the kernel has
@pytest.mark.parametrize("s", [MX, NV], ids=str)
def test_gemm_one_tile(s):
    _run(s, 128, 128, 128 if s.gran == "mx" else 256, seed=800)


@pytest.mark.parametrize("shape", [(128, 256, 512), (256, 384, 1024), (384, 512, 2048), (128, 128, 4096)],
                         ids=lambda t: "x".join(map(str, t)))
@pytest.mark.parametrize("s", [MX, NV, Scheme("e5m2", "mx", layout="gemm")], ids=str)
def test_gemm_shapes(s, shape):
    m, n, k = shape
    _run(s, m, n, k, seed=810 + m + n)


@pytest.mark.parametrize("s", [MX, NV], ids=str)
def test_gemm_bf16_output(s):
    _run(s, 256, 256, 1024, seed=830, dtype=torch.bfloat16)


# more tiles than SMs: CTAs take several tiles in turn (the stage ring runs on across
# them, the accumulator is handed back and forth); 256- and 128-column tiles
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("shape", [(2560, 2048, 512), (1536, 1920, 512)], ids=lambda t: "x".join(map(str, t)))
@pytest.mark.parametrize("s", [MX, NV], ids=str)
def test_gemm_several_tiles_per_cta(s, shape, dtype):
    m, n, k = shape
    _run(s, m, n, k, seed=850 + m + n, dtype=dtype)


@pytest.mark.parametrize("s", [Scheme("e4m3", "mx", hadamard=True, layout="gemm"),
                               Scheme("e2m1", "nv", hadamard=True, layout="gemm")], ids=str)
def test_gemm_rotated_operands(s):
    # both operands rotated by H16/4 along k: the oracle reference is the product of the
    # inverse-rotated (dequantized) operands, which the rotated product equals up to rounding
    a, b = _operands(s, 128, 256, 512, 840)
    qa = bq.quantize(a.cuda(), s, stats=False)
    qb = bq.quantize(b.cuda(), s, stats=False)
    d = bq.gemm(qa, qb)
    torch.cuda.synchronize()
    os_ = _o(s)
    oa = oracle.quantize(synth.bf16_bits(a), os_, stats=False)
    ob = oracle.quantize(synth.bf16_bits(b), os_, stats=False)
    ref = oracle.gemm(oa, ob, 128, 256, 512, os_)
    mag = oracle.gemm_magnitude(oa, ob, 128, 256, 512, os_)
    assert np.all(np.abs(d.cpu().numpy() - ref) <= 1e-3 * mag)


def test_gemm_matches_the_library_gemm():
    # the same MXFP8 operands through cuBLASLt (torch scaled_mm), where this torch has it
    F = torch.nn.functional
    if not (hasattr(F, "scaled_mm") and hasattr(F, "ScalingType") and hasattr(torch, "float8_e8m0fnu")):
        pytest.skip("no block-scaled scaled_mm in this torch")
    a, b = _operands(MX, 256, 384, 2048, 850)
    qa = bq.quantize(a.cuda(), MX, stats=False)
    qb = bq.quantize(b.cuda(), MX, stats=False)
    d = bq.gemm(qa, qb)
    dt = torch.float8_e4m3fn
    try:
        c = F.scaled_mm(qa.codes.view(dt), qb.codes.view(dt).t(),
                        qa.scales.view(torch.float8_e8m0fnu), F.ScalingType.BlockWise1x32,
                        qb.scales.view(torch.float8_e8m0fnu), F.ScalingType.BlockWise1x32,
                        swizzle_a=F.SwizzleType.SWIZZLE_32_4_4, swizzle_b=F.SwizzleType.SWIZZLE_32_4_4,
                        output_dtype=torch.float32)
    except RuntimeError as e:
        pytest.skip(f"library GEMM unavailable for these operands: {e}")
    torch.cuda.synchronize()
    os_ = _o(MX)
    oa = oracle.quantize(synth.bf16_bits(a), os_, stats=False)
    ob = oracle.quantize(synth.bf16_bits(b), os_, stats=False)
    mag = oracle.gemm_magnitude(oa, ob, 256, 384, 2048, os_)
    assert np.all(np.abs(d.cpu().numpy().astype(np.float64) - c.cpu().numpy()) <= 2 * REL * mag)


def _library_nvfp4(qa, qb, out_dtype):
    """D = A B^T through cuBLASLt's NVFP4 GEMM (torch scaled_mm: E2M1 codes, E4M3 block scales
    in the 32x4x4 tile layout, and the two fp32 tensor scales), or None where this torch
    takes no such call."""
    F = torch.nn.functional
    if not (hasattr(F, "scaled_mm") and hasattr(torch, "float4_e2m1fn_x2") and
            hasattr(F.ScalingType, "BlockWise1x16")):
        return None
    fp4, e4 = torch.float4_e2m1fn_x2, torch.float8_e4m3fn
    a, b = qa.codes.view(fp4), qb.codes.view(fp4).t()
    sa, sb = qa.scales.view(e4), qb.scales.view(e4)
    try:
        # two-level form: the block scales and the tensor scale of each operand
        return F.scaled_mm(a, b, [sa, qa.tensor_scale], [F.ScalingType.BlockWise1x16, F.ScalingType.TensorWise],
                           [sb, qb.tensor_scale], [F.ScalingType.BlockWise1x16, F.ScalingType.TensorWise],
                           swizzle_a=[F.SwizzleType.SWIZZLE_32_4_4, F.SwizzleType.NO_SWIZZLE],
                           swizzle_b=[F.SwizzleType.SWIZZLE_32_4_4, F.SwizzleType.NO_SWIZZLE], output_dtype=out_dtype)
    except (RuntimeError, TypeError, ValueError):
        pass
    try:
        # block scales only; the tensor scales multiply the result
        c = F.scaled_mm(a, b, sa, F.ScalingType.BlockWise1x16, sb, F.ScalingType.BlockWise1x16,
                        swizzle_a=F.SwizzleType.SWIZZLE_32_4_4, swizzle_b=F.SwizzleType.SWIZZLE_32_4_4,
                        output_dtype=torch.float32)
        return (c * (qa.tensor_scale * qb.tensor_scale)).to(out_dtype)
    except (RuntimeError, TypeError, ValueError):
        return None


def test_gemm_nvfp4_matches_the_library_gemm():
    # the same NVFP4 operands through cuBLASLt, where this torch has the call
    a, b = _operands(NV, 256, 384, 2048, 860)
    qa = bq.quantize(a.cuda(), NV, stats=False)
    qb = bq.quantize(b.cuda(), NV, stats=False)
    d = bq.gemm(qa, qb)
    c = _library_nvfp4(qa, qb, torch.float32)
    if c is None:
        pytest.skip("no NVFP4 scaled_mm in this torch")
    torch.cuda.synchronize()
    os_ = _o(NV)
    oa = oracle.quantize(synth.bf16_bits(a), os_, stats=False)
    ob = oracle.quantize(synth.bf16_bits(b), os_, stats=False)
    mag = oracle.gemm_magnitude(oa, ob, 256, 384, 2048, os_)
    assert np.all(np.abs(d.cpu().numpy().astype(np.float64) - c.cpu().numpy()) <= 2 * REL * mag)


def test_gemm_argument_checks(cuda_device):
    q = bq.quantize(synth.normal(128, 256, seed=1).cuda(), MX, stats=False)
    d = torch.empty((128, 128), dtype=torch.float32, device=cuda_device)
    row_scales = bq.quantize(synth.normal(128, 256, seed=1).cuda(), Scheme("e4m3", "mx"), stats=False)
    for bad, want in [((row_scales, row_scales), "BQ_ERR_UNSUPPORTED")]:
        with pytest.raises(bq.BqError, match=want):
            bq.bq_gemm(*bad, d)
    i8 = bq.quantize(synth.normal(128, 256, seed=1).cuda(), Scheme("int8_sym", "mx", layout="gemm"), stats=False)
    with pytest.raises(bq.BqError, match="BQ_ERR_UNSUPPORTED"):
        bq.bq_gemm(i8, i8, d)
    assert bq.bq_wait_timeouts() == 0


@pytest.mark.parametrize("s", [MX, NV], ids=str)
def test_gemm_bench_size_sampled(s):
    """The bench's GEMM (8192 x 8192 x 8192, bf16 out, the same operands): every code of
    both operands against the oracle, and 64 sampled rows of D (every column) against the
    oracle's float64 product of those rows."""
    M = N = K = 8192
    a = synth.activations_t3(M, K, seed=2)
    b = synth.weight_outliers(N, K, seed=41)
    qa = bq.quantize(a.cuda(), s, stats=False)
    qb = bq.quantize(b.cuda(), s, stats=False)
    d = bq.gemm(qa, qb, torch.bfloat16)
    torch.cuda.synchronize()
    os_ = _o(s)
    oa = oracle.quantize(synth.bf16_bits(a), os_, stats=False)
    ob = oracle.quantize(synth.bf16_bits(b), os_, stats=False)
    assert np.array_equal(qa.codes.cpu().numpy(), oa["codes"]) and np.array_equal(qb.codes.cpu().numpy(), ob["codes"])
    rows = np.unique(np.concatenate([[0, 127, 128, M - 1], np.random.default_rng(5).choice(M, 60, replace=False)]))
    da = oracle.dequantize(oa["codes"], oa["scales"], None, oa["tensor_scale"], M, K, os_)[rows].astype(np.float64)
    db = oracle.dequantize(ob["codes"], ob["scales"], None, ob["tensor_scale"], N, K, os_).astype(np.float64)
    ref = da @ db.T
    mag = np.abs(da) @ np.abs(db).T
    got = d.float().cpu().numpy()[rows].astype(np.float64)
    bad = np.abs(got - ref) > REL * mag + 2.0 ** -8 * np.abs(ref) + 1e-30
    assert not bad.any(), (s, np.argwhere(bad)[:5])
