"""Seeded synthetic inputs for block-scaled quantization.

This module only draws random numbers and lays them out as bf16 tensors. It holds
none of the quantization arithmetic, and both the CPU oracle (``oracle/``) and the
CUDA library are fed from it, byte for byte.

Every tensor is drawn in float32 from numpy's PCG64 generator with a fixed seed and
rounded to bf16 by torch's round-to-nearest-even cast (a library conversion). The
same seed gives the same bytes on every machine that has the same numpy and torch.

The five workloads stand in for the tensors the source pages measure on (weights
and activations of Llama/Qwen-class models, which are not available here):

* ``tiny_weight``      256 x 1024, N(0, 0.02^2), seed 0 (the small INT4 group
  example of "INT4/INT8/FP8 quantization" §INT4).
* ``weight_outliers``  4096 x 4096, N(0, 0.02^2); 0.1% of the entries (chosen
  without replacement) replaced by a random sign times U(0.1, 0.2), seed 1.
* ``activations_t3``   8192 tokens x 8192 hidden, Student-t(nu=3) * 0.5; 8
  distinct channels rescaled so that their largest |x| is U(100, 200) (the
  "massive activation" outliers of 100-200 named in the 2025 trend article §二),
  seed 2.
* ``ffn_lognormal``    64 tensors of 4096 x 11008 (a Llama-7B FFN weight shape),
  N(0, 1) times a per-row lognormal(0, 0.5) gain, seed 3 + t for tensor t.
* ``weight_x50``       8192 x 28672, N(0, 0.02^2); 0.05% of the entries (chosen
  without replacement) multiplied by 50, seed 4.
"""

from __future__ import annotations

import numpy as np
import torch

__all__ = [
    "WORKLOADS",
    "to_bf16",
    "bf16_bits",
    "normal",
    "uniform",
    "tiny_weight",
    "weight_outliers",
    "activations_t3",
    "ffn_lognormal",
    "weight_x50",
    "workload",
    "random_signs",
    "col_factors",
]


def to_bf16(a: np.ndarray) -> torch.Tensor:
    """float32/float64 numpy array -> contiguous CPU bf16 tensor (torch RNE cast)."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).contiguous()


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """CPU bf16 tensor -> numpy uint16 array of its raw bits (same shape)."""
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def normal(rows: int, cols: int, seed: int, sigma: float = 1.0) -> torch.Tensor:
    """N(0, sigma^2) bf16 tensor [rows, cols]."""
    g = _rng(seed)
    a = g.standard_normal((rows, cols), dtype=np.float32)
    if sigma != 1.0:
        a *= np.float32(sigma)
    return to_bf16(a)


def uniform(rows: int, cols: int, seed: int, lo: float = -1.0, hi: float = 1.0) -> torch.Tensor:
    """U(lo, hi) bf16 tensor [rows, cols]."""
    g = _rng(seed)
    a = g.uniform(lo, hi, size=(rows, cols)).astype(np.float32)
    return to_bf16(a)


def tiny_weight(rows: int = 256, cols: int = 1024, seed: int = 0) -> torch.Tensor:
    return normal(rows, cols, seed, sigma=0.02)


def weight_outliers(rows: int = 4096, cols: int = 4096, seed: int = 1,
                    frac: float = 0.001) -> torch.Tensor:
    g = _rng(seed)
    a = g.standard_normal((rows, cols), dtype=np.float32)
    a *= np.float32(0.02)
    n = rows * cols
    k = int(round(frac * n))
    if k:
        pos = g.choice(n, size=k, replace=False)
        mag = g.uniform(0.1, 0.2, size=k)
        sign = np.where(g.integers(0, 2, size=k) == 0, -1.0, 1.0)
        a.reshape(-1)[pos] = (sign * mag).astype(np.float32)
    return to_bf16(a)


def activations_t3(rows: int = 8192, cols: int = 8192, seed: int = 2,
                   n_outlier_channels: int = 8) -> torch.Tensor:
    g = _rng(seed)
    a = (g.standard_t(3.0, size=(rows, cols)) * 0.5).astype(np.float32)
    nch = min(n_outlier_channels, cols)
    chans = g.choice(cols, size=nch, replace=False)
    targets = g.uniform(100.0, 200.0, size=nch)
    for c, tgt in zip(chans, targets):
        m = float(np.max(np.abs(a[:, c])))
        if m > 0:
            a[:, c] *= np.float32(tgt / m)
    return to_bf16(a)


def ffn_lognormal(t: int, rows: int = 4096, cols: int = 11008, seed0: int = 3) -> torch.Tensor:
    g = _rng(seed0 + t)
    a = g.standard_normal((rows, cols), dtype=np.float32)
    gain = np.exp(0.5 * g.standard_normal(rows)).astype(np.float32)
    a *= gain[:, None]
    return to_bf16(a)


def weight_x50(rows: int = 8192, cols: int = 28672, seed: int = 4,
               frac: float = 0.0005, factor: float = 50.0) -> torch.Tensor:
    g = _rng(seed)
    a = g.standard_normal((rows, cols), dtype=np.float32)
    a *= np.float32(0.02)
    n = rows * cols
    k = int(round(frac * n))
    if k:
        pos = g.choice(n, size=k, replace=False)
        a.reshape(-1)[pos] *= np.float32(factor)
    return to_bf16(a)


def random_signs(n: int, seed: int) -> np.ndarray:
    """n fair coin flips as uint8 0/1 (1 = negate that column), the random diagonal of a
    randomized Hadamard rotation."""
    return _rng(seed).integers(0, 2, size=n, dtype=np.uint8)


def col_factors(n: int, seed: int, sigma: float = 0.5) -> np.ndarray:
    """n positive float32 per-column factors, lognormal(0, sigma): synthetic stand-ins
    for smoothing factors derived from calibration statistics."""
    return np.exp(_rng(seed).normal(0.0, sigma, size=n)).astype(np.float32)


# name -> (generator, full shape, description)
WORKLOADS = {
    "tiny_weight": (tiny_weight, (256, 1024),
                    "bf16 256x1024 N(0,0.02^2) seed 0"),
    "weight_outliers": (weight_outliers, (4096, 4096),
                        "bf16 4096x4096 N(0,0.02^2), 0.1% entries +-U(0.1,0.2), seed 1"),
    "activations_t3": (activations_t3, (8192, 8192),
                       "bf16 8192x8192 t(3)*0.5, 8 channels scaled to max |x| U(100,200), seed 2"),
    "ffn_lognormal": (ffn_lognormal, (4096, 11008),
                      "64 x bf16 4096x11008 N(0,1)*lognormal(0,0.5) row gain, seed 3+t"),
    "weight_x50": (weight_x50, (8192, 28672),
                   "bf16 8192x28672 N(0,0.02^2), 0.05% entries x50, seed 4"),
}


def workload(name: str, **kw) -> torch.Tensor:
    """Generate one tensor of a named workload (``ffn_lognormal`` takes ``t=``)."""
    gen = WORKLOADS[name][0]
    return gen(**kw)
