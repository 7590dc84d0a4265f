"""Pins of the oracle's row transforms (no GPU): the per-column factor of SmoothQuant
("Quantization survey" §3.2, §5.2) and the randomized full-row Hadamard rotation of
QuaRot (same page §5.3: an orthogonal +-1 rotation, R^T R = I, that spreads outlier
channels over the whole row).

* the transform against a dense Sylvester Hadamard matrix (scipy) in float64, within
  the fp32 error bound of log2(n) rounded butterfly stages;
* R^T R = I: energy is kept and the inverse gives the input back (to fp32 rounding);
* n = 16 without signs is the block-16 Hadamard scheme, bit for bit;
* power-of-two factors are exact: quantizing with them equals quantizing the scaled
  bf16 tensor;
* the rotation spreads outlier channels: kappa falls and INT4 per-row QSNR rises.
"""

import math

import numpy as np
import pytest

import oracle
import synth
from oracle import Scheme


def _vals(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32)


@pytest.mark.parametrize("n", [16, 32, 256, 2048, 4096])
def test_rotation_matches_dense_hadamard(n):
    scipy_linalg = pytest.importorskip("scipy.linalg")
    H = scipy_linalg.hadamard(n).astype(np.float64)          # Sylvester order
    rows = 3
    x = synth.bf16_bits(synth.activations_t3(rows, n, seed=60 + n, n_outlier_channels=2))
    m = synth.col_factors(n, seed=61)
    sg = synth.random_signs(n, seed=62)
    y = oracle.rotate_rows(x, col_scale=m, signs=sg)
    xs = (_vals(x) * m).astype(np.float32).astype(np.float64)   # x' = RN(x m)
    sig = np.where(sg != 0, -1.0, 1.0)
    want = (xs * sig) @ H / math.sqrt(n)
    # each output is log2(n) rounded stages of sums, then one rounded product
    bound = (math.log2(n) + 2) * 2.0 ** -24 * (np.abs(xs) @ np.abs(H)) / math.sqrt(n)
    assert np.all(np.abs(y - want) <= bound + 1e-30)
    assert np.max(np.abs(y - want)) > 0 or n == 16          # fp32 rounding is visible


@pytest.mark.parametrize("n", [64, 4096, 16384])
def test_rotation_is_orthogonal(n):
    rows = 4
    x = synth.bf16_bits(synth.normal(rows, n, seed=63, sigma=2.0))
    sg = synth.random_signs(n, seed=64)
    y = oracle.rotate_rows(x, signs=sg)
    xv = _vals(x).astype(np.float64)
    # Parseval: the energy of each row is kept
    assert np.allclose((y.astype(np.float64) ** 2).sum(1), (xv ** 2).sum(1), rtol=1e-5)
    # the inverse (dequantize of an exact code grid is the inverse transform) returns x
    s = Scheme("int8_sym", "row")
    r = oracle.quantize_rt(x, s, signs=sg)
    back = oracle.dequantize_rt(r["codes"], r["scales"], r["zps"], rows, n, s, signs=sg)
    # INT8 per row: the error of every row is at most half a step per rotated element
    step = r["scales"].astype(np.float64)
    err = np.sqrt(((back - xv) ** 2).sum(1))
    assert np.all(err <= 0.5 * step * math.sqrt(n) * 1.001)
    # and the fused sums are the original-domain error
    assert r["stats"][0] == pytest.approx(((back.astype(np.float64) - xv) ** 2).sum(), rel=1e-6)
    assert r["stats"][1] == pytest.approx((xv ** 2).sum(), rel=1e-12)


@pytest.mark.parametrize("s", [Scheme("int8_sym", "row"), Scheme("e4m3", "group", 16), Scheme("int4_sym", "group", 16)], ids=str)
def test_sixteen_points_without_signs_is_block_hadamard(s):
    x = synth.bf16_bits(synth.weight_outliers(8, 16, seed=65))
    a = oracle.quantize_rt(x, s, signs=np.zeros(16, np.uint8))
    b = oracle.quantize(x, Scheme(s.fmt, s.gran, s.block, s.scale_dtype, True))
    assert np.array_equal(a["codes"], b["codes"])
    assert np.array_equal(a["scales"], b["scales"])
    assert a["stats"][0] == b["stats"][0] and a["stats"][1] == b["stats"][1]
    da = oracle.dequantize_rt(a["codes"], a["scales"], a["zps"], 8, 16, s, signs=np.zeros(16, np.uint8))
    db = oracle.dequantize(b["codes"], b["scales"], b["zps"], None, 8, 16, Scheme(s.fmt, s.gran, s.block, s.scale_dtype, True))
    assert np.array_equal(da, db)


@pytest.mark.parametrize("s", [Scheme("uint4_asym", "group", 128, "fp16"), Scheme("int8_sym", "mx"), Scheme("e4m3", "row")], ids=str)
def test_power_of_two_factors_are_exact(s):
    # x * 2^k is exact in bf16: quantizing with the factors equals quantizing the scaled
    # tensor, codes, scales and sums alike
    rows, cols = 6, 512
    x = synth.bf16_bits(synth.weight_outliers(rows, cols, seed=66))
    k = synth._rng(67).integers(-3, 4, size=cols)
    m = np.ldexp(np.ones(cols, np.float32), k).astype(np.float32)
    xs = (_vals(x) * m).view(np.uint32)
    xb = (xs >> 16).astype(np.uint16)
    a = oracle.quantize_rt(x, s, col_scale=m)
    b = oracle.quantize(xb, s)
    assert np.array_equal(a["codes"], b["codes"]) and np.array_equal(a["scales"], b["scales"])
    assert a["stats"][0] == b["stats"][0] and a["stats"][1] == b["stats"][1]
    assert a["stats"][2] == b["stats"][2] and a["stats"][4] == b["stats"][4]


def test_rotation_spreads_outlier_channels():
    # QuaRot's point: a rotation spreads a few outlier channels over the row; per-row
    # kappa falls and INT4 per-row QSNR rises
    rows, cols = 64, 4096
    x = synth.bf16_bits(synth.activations_t3(rows, cols, seed=68, n_outlier_channels=4))
    sg = synth.random_signs(cols, seed=69)
    s = Scheme("int4_sym", "row")
    plain = oracle.quantize_rt(x, s)
    rot = oracle.quantize_rt(x, s, signs=sg)
    k0 = plain["stats"][2] / plain["stats"][4]
    k1 = rot["stats"][2] / rot["stats"][4]
    assert k1 < 0.25 * k0
    assert oracle.qsnr_db(*rot["stats"][:2]) > oracle.qsnr_db(*plain["stats"][:2]) + 10


def test_smoothing_moves_difficulty_to_the_weight():
    # SmoothQuant's factor s_j = sqrt(act_max_j / w_max_j) (alpha = 0.5): activations
    # divided by s lose their outlier channels (INT8 per-token QSNR rises), the weight
    # multiplied by s stays quantizable
    rows, cols = 64, 1024
    act = synth.bf16_bits(synth.activations_t3(rows, cols, seed=70, n_outlier_channels=4))
    w = synth.bf16_bits(synth.normal(rows, cols, seed=71, sigma=0.02))
    a_max = np.abs(_vals(act)).max(0).astype(np.float64)
    w_max = np.abs(_vals(w)).max(0).astype(np.float64)
    f = np.sqrt(a_max / w_max).astype(np.float32)
    s = Scheme("int8_sym", "row")
    plain = oracle.quantize_rt(act, s)
    smoothed = oracle.quantize_rt(act, s, col_scale=(1.0 / f).astype(np.float32))
    assert oracle.qsnr_db(*smoothed["stats"][:2]) > oracle.qsnr_db(*plain["stats"][:2]) + 3
    ws = oracle.quantize_rt(w, s, col_scale=f)
    assert oracle.qsnr_db(*ws["stats"][:2]) > 30


def test_transforms_reject_other_schemes_and_widths():
    x = np.zeros((2, 256), np.uint16)
    for s in [Scheme("int8_sym", "tensor"), Scheme("e2m1", "nv"), Scheme("int8_sym", "row", hadamard=True)]:
        with pytest.raises(ValueError):
            oracle.quantize_rt(x, s, signs=np.zeros(256, np.uint8))
    with pytest.raises(ValueError):
        oracle.quantize_rt(np.zeros((2, 384), np.uint16), Scheme("int8_sym", "row"), signs=np.zeros(384, np.uint8))
    # a factor alone needs no power-of-two width
    oracle.quantize_rt(np.zeros((2, 384), np.uint16), Scheme("int8_sym", "row"), col_scale=np.ones(384, np.float32))
