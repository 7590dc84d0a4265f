"""Pins of the oracle's quantization schemes (no GPU).

* hand-worked tiny tensors (tests/golden/hand_cases.json, each with its page and working);
* invariants the definitions fix: sign symmetry, zero units, the half-step error bound,
  the affine formula, byte counts of 4.25 / 4.5 bit per value;
* the closed-form noise model of "INT vs FP at fine granularity" §4.1
  (QSNR_INT ~ 4.78 + 6.02 b - 20 log10(rho kappa)) and the uniform-noise model for the
  MX and FP8 grids;
* the trends the pages state (uniform data favours INT8 over FP8; Hadamard rotation
  lowers kappa and raises NVINT4 QSNR; MXINT8 beats MXFP8 on Gaussian-like blocks).
"""

import json
import math
import os

import numpy as np
import pytest

import oracle
import synth
from oracle import Scheme

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _hand_cases():
    with open(os.path.join(GOLD, "hand_cases.json")) as f:
        return json.load(f)["cases"]


def _bits_of(values):
    t = synth.to_bf16(np.asarray(values, dtype=np.float32))
    b = synth.bf16_bits(t)
    # hand inputs are exact bf16 values
    assert np.array_equal(t.float().numpy(), np.asarray(values, dtype=np.float32))
    return b


def _scheme(d):
    return Scheme(d["fmt"], d["gran"], d.get("block", 0), d.get("scale_dtype"), d.get("hadamard", False))


@pytest.mark.parametrize("case", _hand_cases(), ids=lambda c: c["name"])
def test_hand_worked_case(case):
    x = _bits_of(case["x"]).reshape(1, -1)
    s = _scheme(case["scheme"])
    r = oracle.quantize(x, s)
    assert r["codes"].reshape(-1).tolist() == case["codes"]
    if "scales_f32" in case:
        assert r["scales"].tolist() == case["scales_f32"]
    if "scales_hex" in case:
        assert [hex(v) for v in r["scales"].view(np.uint32)] == case["scales_hex"]
    if "scales_f16_hex" in case:
        assert [hex(v) for v in r["scales"]] == case["scales_f16_hex"]
    if "zps_f16_hex" in case:
        assert [hex(v) for v in r["zps"]] == case["zps_f16_hex"]
    if "zps_f32" in case:
        assert r["zps"].tolist() == case["zps_f32"]
    if "scales_u8" in case:
        assert r["scales"].tolist() == case["scales_u8"]
    if "tensor_scale_f32" in case:
        assert r["tensor_scale"].tolist() == case["tensor_scale_f32"]
    xh = oracle.dequantize(r["codes"], r["scales"], r["zps"], r["tensor_scale"], 1, x.shape[1], s)
    if "xhat" in case:
        assert xh.reshape(-1).tolist() == case["xhat"]
    if "err2" in case:
        assert r["stats"][0] == case["err2"]
    if "x2" in case:
        assert r["stats"][1] == case["x2"]
    # the standalone sums agree with the fused ones
    st = oracle.qsnr_sums(x, r["codes"], r["scales"], r["zps"], r["tensor_scale"], s)
    assert st[0] == r["stats"][0] and st[1] == r["stats"][1]


def test_hand_case_qsnr_value():
    c = [c for c in _hand_cases() if c["name"] == "int4_sym_group16_ties"][0]
    db = oracle.qsnr_db(c["err2"], c["x2"])
    assert abs(db - 10 * math.log10(2.9453125 / 0.0234375)) < 1e-12
    assert abs(db - 20.9922) < 1e-3


ALL_SCHEMES = [
    Scheme("int8_sym", "tensor"), Scheme("int8_sym", "row"), Scheme("int8_sym", "group", 64),
    Scheme("int8_asym", "tensor"), Scheme("int8_asym", "row"), Scheme("int8_asym", "group", 128, "fp16"),
    Scheme("int4_sym", "group", 64), Scheme("int4_sym", "row"), Scheme("uint4_asym", "group", 128, "fp16"),
    Scheme("e4m3", "tensor"), Scheme("e4m3", "row"), Scheme("e5m2", "tensor"), Scheme("e5m2", "row"),
    Scheme("int8_sym", "mx"), Scheme("e4m3", "mx"), Scheme("e5m2", "mx"), Scheme("e2m1", "mx"),
    Scheme("e2m1", "nv"), Scheme("int4_sym", "nv"), Scheme("int4_sym", "nv", hadamard=True),
    Scheme("e2m1", "nv", hadamard=True), Scheme("int8_sym", "row", hadamard=True),
    Scheme("int8_sym", "tile2d"), Scheme("e4m3", "tile2d"), Scheme("uint4_asym", "tile2d", scale_dtype="fp16"),
]

SYM = [s for s in ALL_SCHEMES if s.fmt not in oracle.ASYM]


@pytest.mark.parametrize("s", SYM, ids=str)
def test_sign_symmetry(s):
    x = synth.bf16_bits(synth.normal(8, 128, seed=11, sigma=0.3))
    xn = x ^ np.uint16(0x8000)
    a = oracle.quantize(x, s)
    b = oracle.quantize(xn, s)
    assert np.array_equal(a["scales"], b["scales"])
    da = oracle.dequantize(a["codes"], a["scales"], a["zps"], a["tensor_scale"], 8, 128, s)
    db = oracle.dequantize(b["codes"], b["scales"], b["zps"], b["tensor_scale"], 8, 128, s)
    assert np.array_equal(da, -db)


@pytest.mark.parametrize("s", ALL_SCHEMES, ids=str)
def test_zero_units_give_zero(s):
    x = synth.bf16_bits(synth.normal(4, 512, seed=12, sigma=0.1))
    x[1, :] = 0        # an all-zero row (a zero unit for every row-local scheme)
    r = oracle.quantize(x, s)
    xh = oracle.dequantize(r["codes"], r["scales"], r["zps"], r["tensor_scale"], 4, 512, s)
    assert np.all(xh[1] == 0.0)
    z = np.zeros((2, 512), np.uint16)
    rz = oracle.quantize(z, s)
    xz = oracle.dequantize(rz["codes"], rz["scales"], rz["zps"], rz["tensor_scale"], 2, 512, s)
    assert np.all(xz == 0.0)
    assert rz["stats"][0] == 0.0 and rz["stats"][1] == 0.0 and rz["stats"][4] == 0.0


@pytest.mark.parametrize("s", [Scheme("int8_sym", "tensor"), Scheme("int8_sym", "row"),
                               Scheme("int4_sym", "group", 64), Scheme("int8_asym", "group", 32),
                               Scheme("uint4_asym", "group", 128, "fp16")], ids=str)
def test_int_error_is_at_most_half_a_step(s):
    x = synth.bf16_bits(synth.uniform(16, 256, seed=13))
    r = oracle.quantize(x, s)
    xh = oracle.dequantize(r["codes"], r["scales"], r["zps"], r["tensor_scale"], 16, 256, s)
    xv = np.array([[oracle.bf16_to_f32(int(b)) for b in row] for row in x], dtype=np.float64)
    unit = {"tensor": 16 * 256, "row": 256}.get(s.gran, s.block)
    sc = r["scales"]
    if sc.dtype == np.uint16:
        sc = np.array([oracle.f16_to_f32(int(v)) for v in sc])
    step = np.repeat(np.asarray(sc, np.float64), unit if s.gran != "tensor" else 16 * 256).reshape(16, 256)
    # half a step, plus the fp32 roundings of the quotient x/s and of the product xhat
    slack = 2.0 ** -22 * (np.abs(xv) + np.abs(xh))
    if s.scale_dtype == "fp16":
        # an fp16 scale is off by up to 2^-11 relative, which the clamped range can reach
        slack = slack + 15 * 2.0 ** -11 * step
    assert np.all(np.abs(xv - xh) <= step / 2 + slack)
    assert np.max(np.abs(xv - xh) / step) > 0.45      # and the bound is nearly reached


def test_affine_formula_on_codes():
    # w = scale * (q - zero_point) for every element (INT4/INT8/FP8 page §INT8)
    s = Scheme("uint4_asym", "group", 128, "fp16")
    x = synth.bf16_bits(synth.weight_outliers(32, 512, seed=21))
    r = oracle.quantize(x, s)
    xh = oracle.dequantize(r["codes"], r["scales"], r["zps"], None, 32, 512, s)
    codes = r["codes"]
    q = np.empty((32, 512), np.int64)
    q[:, 0::2] = codes & 0xF
    q[:, 1::2] = codes >> 4
    sc = np.array([oracle.f16_to_f32(int(v)) for v in r["scales"]], np.float32).reshape(32, 4)
    zp = np.array([oracle.f16_to_f32(int(v)) for v in r["zps"]], np.float32).reshape(32, 4)
    assert np.all((zp >= 0) & (zp <= 15) & (zp == np.round(zp)))
    want = np.repeat(sc, 128, axis=1) * (q - np.repeat(zp, 128, axis=1)).astype(np.float32)
    assert np.array_equal(want.astype(np.float32), xh)


def test_storage_bits_per_value():
    with open(os.path.join(GOLD, "fp_formats.json")) as f:
        g = json.load(f)["storage_bits_per_value"]
    rows, cols = 64, 4096
    c, s, z, t = oracle.buffer_sizes(Scheme("e2m1", "mx"), rows, cols)
    assert (c + s) * 8 / (rows * cols) == g["mxfp4"] and z == 0 and t == 0
    c, s, z, t = oracle.buffer_sizes(Scheme("e2m1", "nv"), rows, cols)
    assert (c + s) * 8 / (rows * cols) == g["nvfp4"] and t * 8 == g["nvfp4_tensor_scale_bits"]
    # INT4: 0.5 byte per parameter
    c, s, z, t = oracle.buffer_sizes(Scheme("int4_sym", "group", 64), rows, cols)
    assert c == rows * cols // 2


def test_invalid_schemes_rejected():
    x = np.zeros((2, 32), np.uint16)
    for s in [Scheme("e2m1", "row"), Scheme("e2m1", "tensor"), Scheme("int8_asym", "mx"),
              Scheme("e4m3", "nv"), Scheme("int8_sym", "group", 48), Scheme("int8_sym", "mx", 16),
              Scheme("int8_sym", "row", scale_dtype="e4m3")]:
        with pytest.raises(ValueError):
            oracle.quantize(x, s)
    with pytest.raises(ValueError):
        oracle.quantize(np.zeros((2, 24), np.uint16), Scheme("int8_sym", "row"))


# --------------------------------------------------------------------------
# closed-form noise models
# --------------------------------------------------------------------------

def _model_db(b, rho, kappa):
    # "INT vs FP at fine granularity" §4.1, with 10 log10(3) = 4.77 and 20 log10(2) = 6.02
    return 10 * math.log10(3) + 20 * math.log10(2) * b - 20 * math.log10(rho * kappa)


def test_page_model_constants():
    with open(os.path.join(GOLD, "fp_formats.json")) as f:
        g = json.load(f)["qsnr_int_model"]
    assert abs(10 * math.log10(3) - g["constant_db"]) < 0.015
    assert abs(20 * math.log10(2) - g["per_bit_db"]) < 0.005


@pytest.mark.parametrize("dist", ["uniform", "normal"])
def test_int8_tensor_qsnr_matches_noise_model(dist):
    n_rows, n_cols = 1024, 1024
    t = synth.uniform(n_rows, n_cols, seed=31) if dist == "uniform" else synth.normal(n_rows, n_cols, seed=32)
    x = synth.bf16_bits(t)
    r = oracle.quantize(x, Scheme("int8_sym", "tensor"))
    err2, x2, kappa = r["stats"][0], r["stats"][1], r["stats"][2]
    got = oracle.qsnr_db(err2, x2)
    amax = float(t.float().abs().max())
    s = float(r["scales"][0])
    rho = s * 2 ** 7 / amax                       # scale precision: 128/127 up to rounding
    assert abs(rho - 128 / 127) < 1e-6
    assert abs(kappa - amax / math.sqrt(x2 / x.size)) < 1e-9
    pred = _model_db(8, rho, kappa)
    assert abs(got - pred) < 0.1, (got, pred)
    if dist == "uniform":
        assert abs(got - 10 * math.log10(4 * 127 ** 2)) < 0.1     # kappa = sqrt(3) closed form


def test_int4_is_about_24db_below_int8_on_uniform():
    x = synth.bf16_bits(synth.uniform(512, 1024, seed=33))
    q8 = oracle.qsnr_db(*oracle.quantize(x, Scheme("int8_sym", "tensor"))["stats"][:2])
    q4 = oracle.qsnr_db(*oracle.quantize(x, Scheme("int4_sym", "tensor"))["stats"][:2])
    # 4 bits fewer: 4 * 6.02 dB, and rho changes from 128/127 to 8/7
    expect = 4 * 20 * math.log10(2) + 20 * math.log10((8 / 7) / (128 / 127))
    assert abs((q8 - q4) - expect) < 1.0


def _grid_msq(n):
    """Mean squared rounding error (in steps) of a value whose fraction takes the n
    equally spaced values k/n, each equally likely, rounded to the nearest integer."""
    k = np.arange(n) / n
    return float(np.mean(np.minimum(k, 1 - k) ** 2))


def test_mxint8_qsnr_matches_uniform_noise_on_each_block_grid():
    # A power-of-two block scale lines the INT grid up with the bf16 grid: a scaled
    # value in [2^j, 2^(j+1)) has 2^(7-j) bf16 points per integer step, so its mean
    # squared error is _grid_msq(2^(7-j)) steps^2 (-> 1/12 for fine bf16 grids).
    t = synth.normal(256, 1024, seed=34)
    x = synth.bf16_bits(t)
    r = oracle.quantize(x, Scheme("int8_sym", "mx"))
    e = np.repeat(r["scales"].astype(np.int64) - 127, 32).reshape(256, 1024)
    v = np.abs(t.float().numpy().astype(np.float64)) * 2.0 ** (-e)
    j = np.floor(np.log2(np.maximum(v, 2.0 ** -40))).astype(np.int64)
    table = {jj: _grid_msq(2 ** (7 - jj)) for jj in range(0, 7)}
    msq = np.array([table.get(jj, 1 / 12) for jj in range(-1, 7)])
    m = np.where(v == 0, 0.0, msq[np.clip(j, -1, 6) + 1])
    noise = np.sum(m * (2.0 ** e) ** 2)
    pred = 10 * math.log10(r["stats"][1] / noise)
    got = oracle.qsnr_db(*r["stats"][:2])
    assert abs(got - pred) < 0.1, (got, pred)
    # the plain 1/12 model is off by the bf16 grid effect, in the stated direction
    noise12 = np.sum(32 * (2.0 ** (r["scales"].astype(np.int64) - 127)) ** 2 / 12)
    assert 10 * math.log10(r["stats"][1] / noise12) > got


@pytest.mark.parametrize("fmt,mbits", [("e4m3", 3), ("e5m2", 2)])
def test_mxfp8_qsnr_matches_uniform_noise_on_the_fp_grid(fmt, mbits):
    t = synth.normal(256, 1024, seed=35)
    x = synth.bf16_bits(t)
    r = oracle.quantize(x, Scheme(fmt, "mx"))
    e = np.repeat(r["scales"].astype(np.int64) - 127, 32).reshape(256, 1024)
    v = np.abs(t.float().numpy().astype(np.float64)) * 2.0 ** (-e)
    emin = {"e4m3": -6, "e5m2": -14}[fmt]
    ex = np.maximum(np.floor(np.log2(np.maximum(v, 1e-300))), emin)
    step = 2.0 ** (ex - mbits) * 2.0 ** e           # grid spacing at each value, original units
    pred = 10 * math.log10(r["stats"][1] / np.sum(step ** 2 / 12))
    got = oracle.qsnr_db(*r["stats"][:2])
    assert abs(got - pred) < 0.3, (got, pred)


# --------------------------------------------------------------------------
# trends the pages state
# --------------------------------------------------------------------------

def test_uniform_data_int8_beats_fp8():
    # "FP8 vs INT8" commentary (youleyou) §3.1: uniform data favours INT8
    x = synth.bf16_bits(synth.uniform(256, 1024, seed=41))
    q8 = oracle.qsnr_db(*oracle.quantize(x, Scheme("int8_sym", "tensor"))["stats"][:2])
    qf = oracle.qsnr_db(*oracle.quantize(x, Scheme("e4m3", "tensor"))["stats"][:2])
    assert q8 > qf + 5


def test_heavier_tails_raise_kappa_and_lower_int8_qsnr():
    xn = synth.bf16_bits(synth.normal(512, 1024, seed=42))
    xt = synth.bf16_bits(synth.activations_t3(512, 1024, seed=43, n_outlier_channels=0))
    rn = oracle.quantize(xn, Scheme("int8_sym", "tensor"))
    rt = oracle.quantize(xt, Scheme("int8_sym", "tensor"))
    assert rt["stats"][2] > rn["stats"][2]
    assert oracle.qsnr_db(*rt["stats"][:2]) < oracle.qsnr_db(*rn["stats"][:2])


def test_hadamard_lowers_kappa_and_raises_nvint4_qsnr():
    # "INT vs FP at fine granularity" §4.2 / §7.2 on weight-like data with x50 outliers
    x = synth.bf16_bits(synth.weight_x50(256, 2048, seed=44, frac=0.0005))
    plain = oracle.quantize(x, Scheme("int4_sym", "nv"))
    rot = oracle.quantize(x, Scheme("int4_sym", "nv", hadamard=True))
    k0 = plain["stats"][2] / plain["stats"][4]
    k1 = rot["stats"][2] / rot["stats"][4]
    assert k1 < k0
    assert oracle.qsnr_db(*rot["stats"][:2]) > oracle.qsnr_db(*plain["stats"][:2])


def test_mxint8_beats_mxfp8_on_gaussian_blocks():
    # "INT vs FP at fine granularity" §4.1/§4.2: block-32 kappa ~ 3 < 7.55, MXINT8 ahead
    x = synth.bf16_bits(synth.ffn_lognormal(0, rows=256, cols=2048))
    ri = oracle.quantize(x, Scheme("int8_sym", "mx"))
    rf = oracle.quantize(x, Scheme("e4m3", "mx"))
    mean_kappa = ri["stats"][2] / ri["stats"][4]
    assert 2.0 < mean_kappa < 7.55
    assert oracle.qsnr_db(*ri["stats"][:2]) > oracle.qsnr_db(*rf["stats"][:2]) + 3


def test_tensor_range_subset_matches_full_call():
    # per-tensor schemes quantize given rows with the whole tensor's range
    x = synth.bf16_bits(synth.activations_t3(64, 256, seed=45, n_outlier_channels=2))
    s = Scheme("e4m3", "tensor")
    full = oracle.quantize(x, s)
    tr = oracle.tensor_range(x)
    part = oracle.quantize(x[10:20], s, tensor_range=tr)
    assert np.array_equal(part["codes"], full["codes"][10:20])
    assert np.array_equal(part["scales"], full["scales"])


def test_clamp_applies_to_the_rounded_quotient_at_any_magnitude():
    # "INT vs FP at fine granularity" §2.1: clip(round(X/s), Qmin, Qmax). An fp16 scale
    # saturates at 65504, so x / s is ~4.6e33 for x ~ 3e38: the codes saturate at
    # +-Qmax with the sign of x.
    big = 1.5 * 2.0 ** 127                                        # exact in bf16
    x = _bits_of([big if i % 2 == 0 else -big for i in range(16)]).reshape(1, 16)
    x = np.ascontiguousarray(x)
    r = oracle.quantize(x, Scheme("int8_sym", "tensor", scale_dtype="fp16"))
    assert r["scales"].tolist() == [0x7BFF]                      # 65504 in fp16
    assert r["codes"].view(np.int8).reshape(-1).tolist() == [127, -127] * 8
    r = oracle.quantize(x, Scheme("int4_sym", "group", 16, "fp16"))
    # INT4 clamps to its full range [-8, 7] ("INT4/INT8/FP8 quantization" §INT4)
    assert r["codes"].reshape(-1).tolist() == [0x87] * 8          # +7 low nibble, -8 high nibble


def test_asymmetric_range_beyond_fp32_saturates():
    # max' - min' overflows fp32 for a unit holding +-3e38: the scale saturates at the
    # largest finite fp32 value (reading), and the codes stay in range.
    vals = [1.5 * 2.0 ** 127, -1.5 * 2.0 ** 127] + [0.0] * 14
    x = _bits_of(vals).reshape(1, 16)
    r = oracle.quantize(np.ascontiguousarray(x), Scheme("int8_asym", "tensor"))
    assert r["scales"].view(np.uint32).tolist() == [0x7F7FFFFF]
    zp = int(r["zps"][0])
    q = r["codes"].view(np.int8).reshape(-1).astype(int)
    assert -128 <= zp <= 127 and q.min() >= -128 and q.max() <= 127


# --------------------------------------------------------------------------
# MXFP6 (E2M3 / E3M2 elements, block 32, UE8M0 scale)
# --------------------------------------------------------------------------

def _ue8m0(amax, qmax):
    """Smallest e with amax <= qmax 2^e, clamped to [-127, 127] (brute force)."""
    if not amax > 0:
        return -127
    for e in range(-300, 300):
        if float(amax) <= float(qmax) * math.ldexp(1.0, e):
            return max(-127, min(127, e))
    raise AssertionError


@pytest.mark.parametrize("fmt,mltype,qmax", [("e2m3", "float6_e2m3fn", 7.5), ("e3m2", "float6_e3m2fn", 28.0)])
def test_mxfp6_blocks_against_ml_dtypes(fmt, mltype, qmax):
    # each block of 32: scale 2^e by the brute-force exponent rule, then the element codes
    # are the library's saturating round-to-nearest-even cast of x / 2^e (an exact scaling)
    ml = pytest.importorskip("ml_dtypes")
    t = getattr(ml, mltype)
    x = synth.bf16_bits(synth.ffn_lognormal(0, rows=16, cols=256))
    vals = np.array([oracle.bf16_to_f32(int(b)) for b in x.reshape(-1)], dtype=np.float32).reshape(x.shape)
    r = oracle.quantize(x, Scheme(fmt, "mx"))
    codes = np.asarray(r["codes"]).reshape(16, 256)
    scales = np.asarray(r["scales"]).reshape(16, 8)
    for i in range(16):
        for b in range(8):
            blk = vals[i, 32 * b:32 * b + 32]
            e = _ue8m0(np.abs(blk).max(), qmax)
            assert int(scales[i, b]) == e + 127
            want = (blk.astype(np.float64) * 2.0 ** (-e)).astype(np.float32).astype(t).view(np.uint8)
            assert np.array_equal(codes[i, 32 * b:32 * b + 32], want), (i, b)


def test_mxfp6_sits_between_mxfp4_and_mxfp8_on_gaussian_blocks():
    # more element mantissa bits, less block error: E2M1 (1 bit) < E2M3 (3 bits) and
    # E3M2 (2 bits) < E2M3; E4M3 (3 bits, wider range) >= E2M3
    x = synth.bf16_bits(synth.ffn_lognormal(0, rows=128, cols=2048))
    db = {f: oracle.qsnr_db(*oracle.quantize(x, Scheme(f, "mx"))["stats"][:2]) for f in ("e2m1", "e3m2", "e2m3", "e4m3")}
    assert db["e2m1"] < db["e3m2"] < db["e2m3"] <= db["e4m3"] + 0.5


def test_fp6_only_with_mx_blocks():
    x = np.zeros((2, 32), np.uint16)
    for s in [Scheme("e2m3", "row"), Scheme("e3m2", "tensor"), Scheme("e2m3", "group", 32), Scheme("e3m2", "nv")]:
        with pytest.raises(ValueError):
            oracle.quantize(x, s)


# --------------------------------------------------------------------------
# 2-D tiles: one scale per 128 x 128 tile ("Quantization survey" §4.4, the DeepSeek-V3
# weight tiles)
# --------------------------------------------------------------------------

TILE2D = [Scheme("int8_sym", "tile2d"), Scheme("e4m3", "tile2d"), Scheme("e5m2", "tile2d", scale_dtype="fp16"),
          Scheme("int8_asym", "tile2d", scale_dtype="fp16"), Scheme("int4_sym", "tile2d"),
          Scheme("uint4_asym", "tile2d", scale_dtype="fp16"), Scheme("e4m3", "tile2d", hadamard=True)]


def _tile_codes(codes, s, r0, r1, c0):
    """Codes of the tile rows r0:r1, columns c0:c0+128 (4-bit codes: 64 bytes)."""
    if s.fmt in oracle.FOUR_BIT:
        return codes[r0:r1, c0 // 2:c0 // 2 + 64]
    return codes[r0:r1, c0:c0 + 128]


@pytest.mark.parametrize("s", TILE2D, ids=str)
def test_tile2d_is_per_tensor_on_each_tile(s):
    # a tile's scale covers exactly its 128 x 128 elements (fewer rows in the last tile
    # row): each tile quantizes as a per-tensor call on that tile alone, whose scheme the
    # hand cases and invariants pin; kappa is the tile's own
    rows, cols = 300, 384                          # tile rows of 128, 128, 44; 3 tile columns
    x = synth.bf16_bits(synth.weight_outliers(rows, cols, seed=71))
    r = oracle.quantize(x, s)
    sdt = r["scales"].dtype
    sc = r["scales"].reshape(3, 3)
    zp = None if r["zps"] is None else r["zps"].reshape(3, 3)
    kap = []
    err2 = 0.0
    for ti, (r0, r1) in enumerate([(0, 128), (128, 256), (256, 300)]):
        for tj in range(3):
            t = np.ascontiguousarray(x[r0:r1, 128 * tj:128 * tj + 128])
            p = oracle.quantize(t, Scheme(s.fmt, "tensor", 0, s.scale_dtype, s.hadamard))
            assert p["scales"].dtype == sdt
            assert p["scales"][0] == sc[ti, tj], (ti, tj)
            if zp is not None:
                assert p["zps"][0] == zp[ti, tj]
            assert np.array_equal(_tile_codes(r["codes"], s, r0, r1, 128 * tj), p["codes"]), (ti, tj)
            kap.append(p["stats"][2])
            err2 += p["stats"][0]
    st = r["stats"]
    assert st[4] == 9
    assert st[3] == pytest.approx(max(kap), rel=1e-12)
    assert st[2] == pytest.approx(sum(kap), rel=1e-12)
    assert st[0] == pytest.approx(err2, rel=1e-9)


def test_tile2d_int8_brute_force():
    # scale = amax / 127 over the 128 x 128 tile in fp32; code = clip(RNE(x / s), +-127)
    rows, cols = 200, 256
    x = synth.bf16_bits(synth.activations_t3(rows, cols, seed=72, n_outlier_channels=3))
    xv = np.array([oracle.bf16_to_f32(int(b)) for b in x.reshape(-1)], np.float32).reshape(rows, cols)
    r = oracle.quantize(x, Scheme("int8_sym", "tile2d"))
    sc = r["scales"].reshape(2, 2)
    q = r["codes"].view(np.int8).reshape(rows, cols).astype(np.int64)
    for ti in range(2):
        for tj in range(2):
            blk = xv[128 * ti:128 * ti + 128, 128 * tj:128 * tj + 128]
            want_s = np.float32(np.abs(blk).max()) / np.float32(127.0)
            assert sc[ti, tj] == want_s
            want_q = np.clip(np.rint(blk / want_s), -127, 127).astype(np.int64)
            assert np.array_equal(q[128 * ti:128 * ti + 128, 128 * tj:128 * tj + 128], want_q)


def test_tile2d_e4m3_against_ml_dtypes():
    # E4M3 elements: the fp32 quotient x / s, then the library's round-to-nearest-even cast
    ml = pytest.importorskip("ml_dtypes")
    rows, cols = 130, 128
    x = synth.bf16_bits(synth.ffn_lognormal(0, rows=rows, cols=cols))
    xv = np.array([oracle.bf16_to_f32(int(b)) for b in x.reshape(-1)], np.float32).reshape(rows, cols)
    r = oracle.quantize(x, Scheme("e4m3", "tile2d"))
    assert r["scales"].shape == (2,)
    for ti, (r0, r1) in enumerate([(0, 128), (128, 130)]):
        blk = xv[r0:r1]
        s = np.float32(np.abs(blk).max()) / np.float32(448.0)
        assert r["scales"][ti] == s
        want = (blk / s).astype(ml.float8_e4m3fn).view(np.uint8)
        assert np.array_equal(r["codes"][r0:r1], want)


def test_tile2d_scale_follows_its_own_tile():
    # multiplying one tile by 2 (exact) doubles its scale and leaves every code and the
    # other tiles' scales unchanged
    rows, cols = 256, 256
    x = synth.bf16_bits(synth.normal(rows, cols, seed=73, sigma=0.5))
    s = Scheme("int8_sym", "tile2d")
    a = oracle.quantize(x, s)
    xv = (x.astype(np.uint32) << 16).view(np.float32)          # bf16 bits to fp32, exact
    xv[128:, :128] *= 2.0                                        # still exact in bf16
    y = (xv.view(np.uint32) >> 16).astype(np.uint16)
    b = oracle.quantize(y, s)
    assert np.array_equal(a["codes"], b["codes"])
    want = a["scales"].copy()
    want[2] *= 2
    assert np.array_equal(b["scales"], want)


def test_tile2d_buffer_sizes_and_dequantize_index():
    s = Scheme("uint4_asym", "tile2d", scale_dtype="fp16")
    c, sb, zb, tb = oracle.buffer_sizes(s, 257, 512)
    assert (c, sb, zb, tb) == (257 * 256, 3 * 4 * 2, 3 * 4 * 2, 0)
    # dequantize: element (r, j) takes the scale and zero point of tile (r // 128, j // 128)
    x = synth.bf16_bits(synth.weight_outliers(257, 512, seed=74))
    r = oracle.quantize(x, s)
    xh = oracle.dequantize(r["codes"], r["scales"], r["zps"], None, 257, 512, s)
    q = np.empty((257, 512), np.int64)
    q[:, 0::2] = r["codes"] & 0xF
    q[:, 1::2] = r["codes"] >> 4
    sc = np.array([oracle.f16_to_f32(int(v)) for v in r["scales"]], np.float32).reshape(3, 4)
    zp = np.array([oracle.f16_to_f32(int(v)) for v in r["zps"]], np.float32).reshape(3, 4)
    ti = np.arange(257)[:, None] // 128
    tj = np.arange(512)[None, :] // 128
    want = sc[ti, tj] * (q - zp[ti, tj]).astype(np.float32)
    assert np.array_equal(want.astype(np.float32), xh)
    st = oracle.qsnr_sums(x, r["codes"], r["scales"], r["zps"], None, s)
    assert st[0] == r["stats"][0] and st[1] == r["stats"][1]


def test_tile2d_rejects_other_shapes():
    x = np.zeros((2, 256), np.uint16)
    for s in [Scheme("e2m1", "tile2d"), Scheme("e2m3", "tile2d"), Scheme("int8_sym", "tile2d", 64),
              Scheme("int8_sym", "tile2d", scale_dtype="ue8m0")]:
        with pytest.raises(ValueError):
            oracle.quantize(x, s)
    with pytest.raises(ValueError):
        oracle.quantize(np.zeros((2, 192), np.uint16), Scheme("int8_sym", "tile2d"))
