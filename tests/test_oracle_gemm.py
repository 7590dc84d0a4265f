"""Pins of the oracle's block-scaled GEMM reference (oracle.gemm): D = A B^T of the
dequantized operands in float64.

- Integer-valued operands that MXFP8 represents exactly (integers in [-8, 8] with an 8 in
  every 32-block: the block exponent is -5 and every x * 2^5 is an E4M3 value) give a
  product equal to the exact integer product, so orientation (B transposed), operand
  order and every scale are pinned by exact integers.
- NVFP4: scaling both inputs by 2^j scales the tensor scales by 2^j and leaves codes and
  block scales alone, so D scales by exactly 2^(2j) (a dropped or doubled tensor scale
  fails), and the result is an NVFP4 product: close to the exact product of the inputs.
"""

import numpy as np

import oracle
import synth


def _int_operand(rows, cols, seed):
    g = np.random.default_rng(seed)
    v = g.integers(-8, 9, size=(rows, cols)).astype(np.float32)
    v[:, ::32] = 8.0 * np.where(g.random((rows, cols // 32)) < 0.5, -1.0, 1.0)
    return v


def test_mxfp8_exact_integer_product():
    s = oracle.Scheme("e4m3", "mx")
    m, n, k = 5, 7, 96
    av, bv = _int_operand(m, k, 1), _int_operand(n, k, 2)
    a = oracle.quantize(synth.bf16_bits(synth.to_bf16(av)), s, stats=False)
    b = oracle.quantize(synth.bf16_bits(synth.to_bf16(bv)), s, stats=False)
    assert np.all(a["scales"] == 127 - 5) and np.all(b["scales"] == 127 - 5)
    d = oracle.gemm(a, b, m, n, k, s)
    want = av.astype(np.int64) @ bv.astype(np.int64).T
    assert d.shape == (m, n)
    assert np.array_equal(d, want.astype(np.float64))
    # E5M2 represents them exactly too (block exponent -12: x * 2^12 has at most 3 significant bits)
    s5 = oracle.Scheme("e5m2", "mx")
    a5 = oracle.quantize(synth.bf16_bits(synth.to_bf16(av)), s5, stats=False)
    b5 = oracle.quantize(synth.bf16_bits(synth.to_bf16(bv)), s5, stats=False)
    assert np.array_equal(oracle.gemm(a5, b5, m, n, k, s5), want.astype(np.float64))


def test_nvfp4_power_of_two_scaling_and_closeness():
    s = oracle.Scheme("e2m1", "nv")
    m, n, k = 4, 6, 256
    g = np.random.default_rng(3)
    av = g.standard_normal((m, k)).astype(np.float32)
    bv = g.standard_normal((n, k)).astype(np.float32)

    def run(scale):
        a = oracle.quantize(synth.bf16_bits(synth.to_bf16(av * scale)), s, stats=False)
        b = oracle.quantize(synth.bf16_bits(synth.to_bf16(bv * scale)), s, stats=False)
        return a, b, oracle.gemm(a, b, m, n, k, s)

    a1, b1, d1 = run(1.0)
    a8, b8, d8 = run(8.0)
    assert np.array_equal(a1["codes"], a8["codes"]) and np.array_equal(a1["scales"], a8["scales"])
    assert a8["tensor_scale"][0] == 8.0 * a1["tensor_scale"][0]
    assert np.array_equal(d8, 64.0 * d1)
    # an NVFP4 product of N(0, 1) rows: within a few percent of the exact inputs' product
    ax = synth.bf16_bits(synth.to_bf16(av)).astype(np.uint32) << 16
    bx = synth.bf16_bits(synth.to_bf16(bv)).astype(np.uint32) << 16
    exact = ax.view(np.float32).astype(np.float64) @ bx.view(np.float32).astype(np.float64).T
    mag = np.abs(ax.view(np.float32)).astype(np.float64) @ np.abs(bx.view(np.float32)).astype(np.float64).T
    assert np.all(np.abs(d1 - exact) <= 0.25 * mag)
    assert np.max(np.abs(d1 - exact) / mag) > 0.0          # FP4 is not exact
