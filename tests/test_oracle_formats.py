"""Pins of the oracle's number formats against what the pages and libraries fix.

No GPU. Every check here compares the oracle with something other than itself: the
page constants in tests/golden/fp_formats.json, exhaustive enumeration, the round to
nearest even rule worked by hand, torch's float8 casts, torch's bf16 cast, numpy's
float16 cast, scipy's Hadamard matrix, and a brute-force search for the UE8M0 exponent.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _formats():
    with open(os.path.join(GOLD, "fp_formats.json")) as f:
        return json.load(f)


@pytest.mark.parametrize("fmt,nbits,n_finite", [("e4m3", 8, 254), ("e5m2", 8, 248), ("e2m1", 4, 16)])
def test_page_constants_and_finite_code_count(fmt, nbits, n_finite):
    g = _formats()[fmt]
    vals = [oracle.fp_decode(fmt, c) for c in range(1 << nbits)]
    finite = [v for v in vals if math.isfinite(v)]
    assert len(finite) == n_finite
    assert max(finite) == g["max"] and min(finite) == -g["max"]
    pos = [v for v in finite if v > 0]
    assert min(pos) == g["min_positive_exact"]
    # the page's rounded figure names that power of two
    assert abs(min(pos) - g["min_positive_approx"]) / g["min_positive_exact"] < 0.05


def test_e2m1_value_set():
    vals = sorted(oracle.fp_decode("e2m1", c) for c in range(8))
    assert vals == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert [oracle.fp_decode("e2m1", c | 8) for c in range(8)] == [-v for v in
                                                                   [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]]


def test_bit_layout_fields():
    # [s][eeee][mmm]: 1.0 has exponent field = bias 7 -> 0b0_0111_000
    assert oracle.fp_decode("e4m3", 0b0_0111_000) == 1.0
    assert oracle.fp_decode("e4m3", 0b1_1000_100) == -3.0     # -(1 + 4/8) * 2^1
    # [s][eeeee][mm]: bias 15
    assert oracle.fp_decode("e5m2", 0b0_01111_00) == 1.0
    assert oracle.fp_decode("e5m2", 0b0_10001_11) == 7.0      # (1 + 3/4) * 2^2
    # [s][ee][m]: bias 1
    assert oracle.fp_decode("e2m1", 0b0_10_1) == 3.0
    # E4M3 is the FN variant: only S.1111.111 is NaN; E5M2 keeps IEEE inf/NaN
    assert math.isnan(oracle.fp_decode("e4m3", 0x7F)) and math.isnan(oracle.fp_decode("e4m3", 0xFF))
    assert oracle.fp_decode("e4m3", 0x7E) == 448.0
    assert oracle.fp_decode("e5m2", 0x7C) == math.inf
    assert math.isnan(oracle.fp_decode("e5m2", 0x7D))


@pytest.mark.parametrize("fmt,nbits", [("e4m3", 8), ("e5m2", 8), ("e2m1", 4)])
def test_exhaustive_round_trip(fmt, nbits):
    for c in range(1 << nbits):
        v = oracle.fp_decode(fmt, c)
        if not math.isfinite(v):
            continue
        assert oracle.fp_encode(fmt, v) == c, (fmt, hex(c), v)


def test_e2m1_ties_and_saturation_by_hand():
    # ties go to the even mantissa; beyond 6 saturates (round to nearest even rule)
    cases = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0, 7.0: 6.0,
             100.0: 6.0, 0.26: 0.5, 0.74: 0.5, 4.9: 4.0, 5.1: 6.0}
    for v, want in cases.items():
        assert oracle.fp_decode("e2m1", oracle.fp_encode("e2m1", v)) == want, v
        assert oracle.fp_decode("e2m1", oracle.fp_encode("e2m1", -v)) == -want, -v


def test_e4m3_saturates_not_nan_and_keeps_sign_of_zero():
    assert oracle.fp_encode("e4m3", 464.0) == 0x7E
    assert oracle.fp_encode("e4m3", 1e30) == 0x7E
    assert oracle.fp_encode("e4m3", -1e30) == 0xFE
    assert oracle.fp_encode("e4m3", 2.0 ** -10) == 0x00
    assert oracle.fp_encode("e4m3", -(2.0 ** -10)) == 0x80
    assert oracle.fp_encode("e4m3", -0.0) == 0x80
    assert oracle.fp_encode("e5m2", 1e30) == 0x7B
    assert oracle.fp_encode("e5m2", 61440.0) == 0x7B


def _fp8_candidates(fmt):
    """Random fp32 values plus every midpoint between neighbours and its two fp32 neighbours."""
    mx = _formats()[fmt]["max"]
    vals = sorted({oracle.fp_decode(fmt, c) for c in range(256) if math.isfinite(oracle.fp_decode(fmt, c))})
    out = []
    for a, b in zip(vals[:-1], vals[1:]):
        m = np.float32((a + b) / 2)
        out += [m, np.nextafter(m, np.float32(np.inf)), np.nextafter(m, np.float32(-np.inf))]
    g = np.random.default_rng(7)
    out += list((g.standard_normal(20000) * mx / 8).astype(np.float32))
    out += list((g.uniform(-1, 1, 20000) * 2.0 ** g.integers(-30, 20, 20000)).astype(np.float32))
    a = np.array(out, dtype=np.float32)
    return np.clip(a, -mx, mx)


@pytest.mark.parametrize("fmt,tdt", [("e4m3", torch.float8_e4m3fn), ("e5m2", torch.float8_e5m2)])
def test_fp8_encoder_matches_torch_cast(fmt, tdt):
    # torch's float -> float8 casts round to nearest even; they do not saturate, so
    # the inputs are clamped to the finite range first.
    a = _fp8_candidates(fmt)
    ref = torch.from_numpy(a).to(tdt).view(torch.uint8).numpy()
    mine = np.array([oracle.fp_encode(fmt, float(v)) for v in a], dtype=np.uint8)
    bad = np.nonzero(ref != mine)[0]
    assert bad.size == 0, [(float(a[i]), hex(ref[i]), hex(mine[i])) for i in bad[:5]]


def test_bf16_rounding_matches_torch():
    g = np.random.default_rng(3)
    bits = g.integers(0, 2 ** 32, 200000, dtype=np.uint64).astype(np.uint32)
    f = bits.view(np.float32)
    f = f[np.isfinite(f)]
    f = f[np.abs(f) < 3.0e38]
    # include exact ties on the dropped half
    ties = (g.integers(0, 2 ** 16, 5000, dtype=np.uint64).astype(np.uint32) << 16 | 0x8000).view(np.float32)
    ties = ties[np.isfinite(ties) & (np.abs(ties) < 3.0e38)]
    f = np.concatenate([f, ties, np.array([0.0, -0.0, 1e-45, -1e-45], dtype=np.float32)])
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    mine = oracle.to_bf16_array(f)
    assert np.array_equal(ref, mine)
    assert oracle.bf16_to_f32(0x3F80) == 1.0 and oracle.bf16_to_f32(0xC040) == -3.0


def test_fp16_rounding_matches_numpy():
    g = np.random.default_rng(4)
    f = np.concatenate([
        (g.standard_normal(50000) * 10.0 ** g.integers(-8, 5, 50000)).astype(np.float32),
        np.array([65504.0, 65519.0, 2.0 ** -24, 2.0 ** -25, 1.5 * 2.0 ** -25, 0.1], dtype=np.float32),
    ])
    ref = f.astype(np.float16).view(np.uint16)
    mine = np.array([oracle.f32_to_f16(float(v)) for v in f], dtype=np.uint16)
    assert np.array_equal(ref, mine)
    assert oracle.f16_to_f32(0x3C00) == 1.0


def _ue8m0_brute(amax, qmax):
    if not amax > 0:
        return -127
    a, q = float(amax), float(qmax)
    for e in range(-300, 300):
        if a <= q * math.ldexp(1.0, e):
            return max(-127, min(127, e))
    raise AssertionError


def test_ue8m0_exponent_is_smallest_e_with_amax_le_qmax_2e():
    g = np.random.default_rng(5)
    amaxes = list((g.uniform(0.5, 2.0, 3000) * 2.0 ** g.integers(-140, 120, 3000)).astype(np.float32))
    for q in (127.0, 448.0, 57344.0, 6.0):
        edges = []
        for e in range(-130, 110, 7):
            v = np.float32(q * 2.0 ** e)
            edges += [v, np.nextafter(v, np.float32(np.inf)), np.nextafter(v, np.float32(0))]
        for a in amaxes + edges + [np.float32(0.0), np.float32(1e-45)]:
            assert oracle.ue8m0_exponent(float(a), q) == _ue8m0_brute(a, q), (a, q)


def test_fwht16_matches_hadamard_matrix_and_is_an_involution():
    from scipy.linalg import hadamard
    H = hadamard(16).astype(np.float64)
    assert np.array_equal(H @ H, 16 * np.eye(16))
    g = np.random.default_rng(6)
    for _ in range(50):
        x = g.integers(-1000, 1000, 16).astype(np.float32)
        y = oracle.fwht16(x)
        assert np.array_equal(y.astype(np.float64), H @ x.astype(np.float64) / 4.0)   # exact on integers
        assert np.array_equal(oracle.fwht16(y), x)
    x = g.standard_normal(16).astype(np.float32)
    assert np.allclose(oracle.fwht16(x), H @ x / 4.0, rtol=0, atol=1e-6)
    one = np.zeros(16, np.float32)
    one[0] = 1.0
    assert np.array_equal(oracle.fwht16(one), np.full(16, 0.25, np.float32))
    two = np.zeros(16, np.float32)
    two[:2] = 1.0
    assert np.array_equal(oracle.fwht16(two), np.tile(np.array([0.5, 0.0], np.float32), 8))


# --- FP6 (MXFP6 element formats) -------------------------------------------------

@pytest.mark.parametrize("fmt", ["e2m3", "e3m2"])
def test_fp6_page_range_and_code_count(fmt):
    g = _formats()[fmt]
    vals = [oracle.fp_decode(fmt, c) for c in range(64)]
    assert all(math.isfinite(v) for v in vals)          # no inf / NaN codes
    assert max(vals) == g["max"] and min(vals) == -g["max"]
    # the page's smallest positive value contradicts its range; the range's bias wins
    assert min(v for v in vals if v > 0) == g["min_positive_of_the_range"]
    assert min(v for v in vals if v > 0) != g["page_min_positive"]


@pytest.mark.parametrize("fmt,mltype", [("e2m3", "float6_e2m3fn"), ("e3m2", "float6_e3m2fn")])
def test_fp6_decode_and_encode_against_ml_dtypes(fmt, mltype):
    ml = pytest.importorskip("ml_dtypes")
    t = getattr(ml, mltype)
    codes = np.arange(64, dtype=np.uint8)
    lib_vals = codes.view(t).astype(np.float32)
    assert [oracle.fp_decode(fmt, int(c)) for c in codes] == [float(v) for v in lib_vals]
    # every midpoint between neighbours, its fp32 neighbours, values past the range, and
    # random values: the library's round-to-nearest-even cast (saturating) must agree
    pos = sorted(set(float(v) for v in lib_vals if v >= 0))
    cand = []
    for a, b in zip(pos[:-1], pos[1:]):
        m = np.float32((a + b) / 2)
        cand += [m, np.nextafter(m, np.float32(np.inf)), np.nextafter(m, np.float32(-np.inf))]
    g = np.random.default_rng(11)
    cand += list(g.uniform(-1.2 * pos[-1], 1.2 * pos[-1], 4000).astype(np.float32))
    cand += [np.float32(pos[-1] * 4), np.float32(1e30), np.float32(-0.0)]
    cand = np.array(cand, dtype=np.float32)
    cand = np.concatenate([cand, -cand])
    want = cand.astype(t).view(np.uint8)
    got = np.array([oracle.fp_encode(fmt, float(v)) for v in cand], dtype=np.uint8)
    assert np.array_equal(got, want)


@pytest.mark.parametrize("fmt", ["e2m3", "e3m2"])
def test_fp6_exhaustive_round_trip(fmt):
    for c in range(64):
        assert oracle.fp_encode(fmt, oracle.fp_decode(fmt, c)) == c, (fmt, hex(c))
