"""bq_quantize_batch on the GPU: a batch of same-shape tensors in one launch.

Each tensor's codes, scales and zero points must equal the oracle's for that tensor (and
so bq_quantize's) bit for bit; its QSNR and kappa sums match the oracle within the parity
tolerances (1e-5 relative; QSNR 0.01 dB). At full size: the 64 FFN tensors of 4096 x 11008
under MXINT8 and MXFP8, every tensor against the one-tensor call, tensors 0 and 63
against the oracle.
"""

import math

import numpy as np
import pytest
import torch

import oracle
import synth
import block_scaled_bit_bq_b200 as bq
from block_scaled_bit_bq_b200 import Scheme

pytestmark = pytest.mark.gpu

SUM_RTOL = 1e-5


def _o(s):
    return oracle.Scheme(s.fmt, s.gran, s.block, s.scale_dtype, s.hadamard)


def _close(a, b, rtol=SUM_RTOL, atol=1e-30):
    if math.isinf(a) or math.isinf(b):
        return a == b
    return abs(a - b) <= atol + rtol * max(abs(a), abs(b))


def _bytes(t):
    return t.detach().cpu().contiguous().view(torch.uint8).numpy().reshape(-1)


def _check_tensor(q: bq.QuantizedBatch, b: int, xb: np.ndarray, s: Scheme, what: str):
    o = oracle.quantize(xb, _o(s))
    assert np.array_equal(q.codes[b].cpu().numpy(), o["codes"]), f"{what} tensor {b}: codes"
    assert np.array_equal(_bytes(q.scales[b]), o["scales"].view(np.uint8).reshape(-1)) or \
        s.layout == "gemm", f"{what} tensor {b}: scales"
    if o["zps"] is not None:
        assert np.array_equal(_bytes(q.zero_points[b]), o["zps"].view(np.uint8).reshape(-1)), f"{what} {b}: zps"
    st = q.stats[b].cpu().numpy()
    ost = o["stats"]
    assert _close(st[1], ost[1]) and _close(st[0], ost[0], atol=1e-30 + 1e-7 * ost[1]), (what, b, st, ost)
    if ost[0] > 0:
        assert abs(bq.bq_stats_to_db(st) - oracle.qsnr_db(ost[0], ost[1])) < 0.01
    assert st[4] == ost[4] and _close(st[2], ost[2]) and _close(st[3], ost[3]), (what, b, st, ost)
    return o


SCHEMES = [Scheme("int8_sym", "mx"), Scheme("e4m3", "mx"), Scheme("e2m1", "mx"), Scheme("e2m3", "mx", hadamard=True),
           Scheme("e4m3", "mx", layout="gemm"),
           Scheme("int4_sym", "group", 64), Scheme("uint4_asym", "group", 128, "fp16"), Scheme("int8_asym", "group", 32),
           Scheme("e5m2", "group", 16, "fp16"), Scheme("int8_sym", "group", 512), Scheme("int8_sym", "row"),
           Scheme("uint4_asym", "row", scale_dtype="fp16")]


@pytest.mark.parametrize("shape", [(3, 128, 1024), (5, 36, 512), (2, 256, 2048), (9, 1, 64 * 8)],
                         ids=lambda t: "x".join(map(str, t)))
@pytest.mark.parametrize("s", SCHEMES, ids=str)
def test_batch_parity_small(s, shape, cuda_device):
    B, rows, cols = shape
    try:
        oracle.buffer_sizes(_o(s), rows, cols)
    except ValueError:
        pytest.skip("scheme does not divide this shape")
    if s.layout == "gemm" and (rows % 128 or cols % 128):
        pytest.skip("GEMM-layout batches need rows % 128 == 0")
    if s.gran == "row" and cols > 2048:
        pytest.skip("per-row batches: cols up to 2048")
    xs = [synth.activations_t3(rows, cols, seed=700 + 13 * b + rows, n_outlier_channels=2) for b in range(B)]
    x = torch.stack(xs).to(cuda_device)
    ws = bq.new_workspace(cuda_device)
    q = bq.quantize_batch(x, s, workspace=ws)
    q2 = bq.quantize_batch(x, s, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(q.stats, q2.stats)                      # fixed reduction order
    for b in range(B):
        o = _check_tensor(q, b, synth.bf16_bits(xs[b]), s, f"{s} {shape}")
        single = bq.quantize(xs[b].to(cuda_device), s, workspace=ws)
        torch.cuda.synchronize()
        assert torch.equal(single.codes, q.codes[b]) and torch.equal(single.scales.view(-1), q.scales[b])
        if s.layout == "gemm":
            nb = cols // 32
            got = q.scales[b].cpu().numpy().view(np.uint8)
            assert np.array_equal(oracle.scales_from_gemm(got, rows, nb), o["scales"].reshape(rows, nb))


def test_batch_of_one_and_empty(cuda_device):
    s = Scheme("int8_sym", "mx")
    x = synth.ffn_lognormal(5, rows=64, cols=1024).to(cuda_device)
    ws = bq.new_workspace(cuda_device)
    q = bq.quantize_batch(x[None], s, workspace=ws)
    ref = bq.quantize(x, s, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(q.codes[0], ref.codes) and torch.equal(q.stats[0], ref.stats)
    # zero tensors: nothing to do; empty tensors: zeroed stats
    bq.bq_quantize_batch(torch.empty((0, 4, 64), dtype=torch.bfloat16, device=cuda_device), s,
                         q.codes, q.scales, None, q.stats, ws)
    e = bq.alloc_batch_outputs(s, 3, 0, 64, cuda_device)
    e.stats.fill_(7.0)
    bq.bq_quantize_batch(torch.empty((3, 0, 64), dtype=torch.bfloat16, device=cuda_device), s,
                         e.codes, e.scales, None, e.stats, ws)
    torch.cuda.synchronize()
    assert e.stats.abs().sum().item() == 0.0


@pytest.mark.parametrize("s", [Scheme("int8_sym", "mx"), Scheme("e4m3", "mx"), Scheme("e4m3", "mx", layout="gemm")],
                         ids=str)
def test_ffn_batch_full(s, cuda_device):
    """The 64 FFN tensors of 4096 x 11008 in one call (the bench's launch; with GEMM-layout
    scales the call runs as several launches of at most 16 MiB of scales): every tensor
    against the one-tensor call; tensors 0 and 63 against the oracle."""
    from concurrent.futures import ThreadPoolExecutor
    with ThreadPoolExecutor(8) as ex:
        hosts = list(ex.map(synth.ffn_lognormal, range(64)))
    x = torch.empty((64, 4096, 11008), dtype=torch.bfloat16, device=cuda_device)
    for t, h in enumerate(hosts):
        x[t].copy_(h)
    ws = bq.new_workspace(cuda_device)
    q = bq.quantize_batch(x, s, workspace=ws)
    torch.cuda.synchronize()
    one = bq.alloc_outputs(s, 4096, 11008, cuda_device)
    for t in range(64):
        bq.quantize(x[t], s, workspace=ws, out=one)
        torch.cuda.synchronize()
        assert torch.equal(one.codes, q.codes[t]), t
        assert torch.equal(one.scales.view(-1), q.scales[t]), t
        a, b = one.stats.cpu().tolist(), q.stats[t].cpu().tolist()
        assert abs(bq.bq_stats_to_db(a) - bq.bq_stats_to_db(b)) < 1e-6 and a[4] == b[4], (t, a, b)
    for t in (0, 63):
        _check_tensor(q, t, synth.bf16_bits(hosts[t]), s, "ffn batch")
