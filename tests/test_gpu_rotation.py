"""GPU parity of the row transforms (per-column factor, randomized full-row Hadamard
rotation) against the oracle: codes, scales and zero points bit-exact, the inverse
rotation's dequantized values bit-exact (fp32 and bf16), QSNR within 0.01 dB, kappa
and the sums within 1e-5 (the fused sums are taken on the rotated values, the
oracle's against x'; the rotation is orthogonal, so they agree to rounding)."""

import math

import numpy as np
import pytest
import torch

import oracle
import synth
import block_scaled_bit_bq_b200 as bq
from block_scaled_bit_bq_b200 import Scheme

pytestmark = pytest.mark.gpu

SCHEMES = [Scheme("int8_sym", "row"), Scheme("uint4_asym", "group", 128, "fp16"), Scheme("int4_sym", "group", 64),
           Scheme("e4m3", "group", 128), Scheme("int8_asym", "row", scale_dtype="fp16"), Scheme("int8_sym", "mx"),
           Scheme("e2m1", "mx"), Scheme("e5m2", "group", 16), Scheme("e2m3", "mx")]

SHAPES = [(37, 4096), (9, 512), (5, 16384), (300, 2048), (203, 1024), (2501, 2048)]
TRANSFORMS = ["signs", "factor", "both", "none"]


def _o(s):
    return oracle.Scheme(s.fmt, s.gran, s.block, s.scale_dtype, s.hadamard)


def _bytes(t):
    if isinstance(t, torch.Tensor):
        return t.detach().cpu().contiguous().view(torch.uint8).numpy().reshape(-1)
    return np.ascontiguousarray(t).view(np.uint8).reshape(-1)


def _close(a, b, rtol=1e-5):
    return abs(a - b) <= 1e-30 + rtol * max(abs(a), abs(b))


def _transforms(kind, cols, seed):
    signs = synth.random_signs(cols, seed) if kind in ("signs", "both") else None
    factor = synth.col_factors(cols, seed + 1) if kind in ("factor", "both") else None
    return signs, factor


@pytest.fixture(scope="module")
def ws(cuda_device):
    return bq.new_workspace(cuda_device)


def check_rt(x, s, signs, factor, ws, what=""):
    rows, cols = x.shape
    xb = synth.bf16_bits(x)
    dev = torch.device("cuda")
    sb = None if signs is None else bq.pack_sign_bits(signs, dev)
    cs = None if factor is None else torch.from_numpy(factor).to(dev)
    q = bq.quantize_rt(x.to(dev), s, col_scale=cs, sign_bits=sb, stats=True, workspace=ws)
    d32 = bq.dequantize_rt(q, cs, sb, torch.float32)
    d16 = bq.dequantize_rt(q, cs, sb, torch.bfloat16)
    torch.cuda.synchronize()
    o = oracle.quantize_rt(xb, _o(s), col_scale=factor, signs=signs)
    oxh = oracle.dequantize_rt(o["codes"], o["scales"], o["zps"], rows, cols, _o(s), signs=signs)
    codes = q.codes.cpu().numpy()
    assert np.array_equal(codes, o["codes"]), f"{what} {s}: codes differ at {np.argwhere(codes != o['codes'])[:5]}"
    assert np.array_equal(_bytes(q.scales), _bytes(o["scales"])), f"{what} {s}: scales"
    if o["zps"] is not None:
        assert np.array_equal(_bytes(q.zero_points), _bytes(o["zps"])), f"{what} {s}: zero points"
    g = d32.cpu().numpy()
    bad = np.nonzero(g.view(np.uint32) != oxh.view(np.uint32))
    assert bad[0].size == 0, f"{what} {s}: fp32 dequant differs at {list(zip(*bad))[:5]}"
    assert np.array_equal(_bytes(d16).view(np.uint16), oracle.to_bf16_array(oxh).reshape(-1)), f"{what} {s}: bf16"
    st = q.stats.cpu().numpy()
    ost = o["stats"]
    assert _close(st[1], ost[1]) and _close(st[0], ost[0]), (what, s, st, ost)
    if ost[0] > 0:
        assert abs(bq.bq_stats_qsnr_db(st) - oracle.qsnr_db(ost[0], ost[1])) < 0.01
    assert st[4] == ost[4] and _close(st[2], ost[2]) and _close(st[3], ost[3]), (what, s, st, ost)


@pytest.mark.parametrize("kind", TRANSFORMS)
@pytest.mark.parametrize("shape", SHAPES, ids=lambda t: f"{t[0]}x{t[1]}")
@pytest.mark.parametrize("s", SCHEMES, ids=str)
def test_rt_parity(s, shape, kind, ws):
    rows, cols = shape
    x = synth.activations_t3(rows, cols, seed=400 + rows, n_outlier_channels=3)
    signs, factor = _transforms(kind, cols, 500 + cols)
    check_rt(x, s, signs, factor, ws, f"{kind} {rows}x{cols}")


def test_rt_edge_values(ws):
    # zero rows, tiny and huge values (whole rows and half rows), exact ties under
    # power-of-two factors
    g = np.random.default_rng(9)
    a = (g.standard_t(3, size=(6, 1024)) * 0.5).astype(np.float32)
    a[0] = 0.0
    a[1] *= 1e-30
    a[2] = g.uniform(-1, 1, 1024).astype(np.float32) * 1e30
    a[3] = g.integers(-64, 65, 1024).astype(np.float32) * 0.5
    a[4, 512:] *= 1e-30          # units of one row (and of one warp) on both sides of
    a[5, :512] *= 1e30           # the plain-sums range: the scaled and unscaled forms mix
    x = synth.to_bf16(a)
    signs = synth.random_signs(1024, 7)
    factor = np.ldexp(np.ones(1024, np.float32), g.integers(-2, 3, 1024)).astype(np.float32)
    for s in [Scheme("int8_sym", "row"), Scheme("uint4_asym", "group", 64, "fp16"), Scheme("e4m3", "mx")]:
        check_rt(x, s, signs, factor, ws, "edge")
        check_rt(x, s, signs, None, ws, "edge")
        check_rt(x, s, None, factor, ws, "edge, no rotation")


def test_rt_full_size_weight(ws):
    # the 4096 x 4096 outlier weight, MXFP4 and INT4 per-group with the rotation
    x = synth.weight_outliers()
    signs = synth.random_signs(4096, 11)
    for s in [Scheme("e2m1", "mx"), Scheme("int4_sym", "group", 128)]:
        check_rt(x, s, signs, None, ws, "weight_outliers")


def test_rt_rotation_raises_int4_qsnr_on_outlier_channels(ws):
    x = synth.activations_t3(256, 4096, seed=12, n_outlier_channels=8).cuda()
    sb = bq.pack_sign_bits(synth.random_signs(4096, 13), x.device)
    s = Scheme("int4_sym", "row")
    plain = bq.quantize_rt(x, s, workspace=ws)
    rot = bq.quantize_rt(x, s, sign_bits=sb, workspace=ws)
    assert rot.qsnr_db() > plain.qsnr_db() + 10
    assert rot.mean_kappa() < 0.25 * plain.mean_kappa()


def test_rt_empty(ws, cuda_device):
    s = Scheme("int8_sym", "row")
    x = torch.empty((0, 512), dtype=torch.bfloat16, device=cuda_device)
    q = bq.alloc_outputs(s, 0, 512, cuda_device)
    q.stats.fill_(7.0)
    bq.bq_quantize_rt(x, s, None, None, q.codes, q.scales, q.zero_points, q.stats, ws)
    torch.cuda.synchronize()
    assert q.stats.cpu().tolist() == [0.0] * 5
