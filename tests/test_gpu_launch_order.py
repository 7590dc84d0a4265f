"""Stream order across back-to-back launches.

The quantize, dequantize and QSNR kernels go out with programmatic dependent launch: a
launch may be scheduled while the kernel ahead of it in the stream is finishing, and waits
for it to complete before touching global memory. Each case here makes the kernel ahead
of a call the one that writes that call's input (read after write), or the one that reads
what the call overwrites (write after read), with no synchronisation in between, eagerly
and inside a CUDA graph, and checks every result against the oracle.
"""

import numpy as np
import pytest
import torch

import oracle
import synth
import block_scaled_bit_bq_b200 as bq
from block_scaled_bit_bq_b200 import Scheme

pytestmark = pytest.mark.gpu

# two-pass (per-tensor, NV: range pass, then quantize pass through the workspace) and
# one-pass schemes, flat and per-row kernels
SCHEMES = [Scheme("int8_sym", "mx"), Scheme("e4m3", "tensor"), Scheme("e2m1", "nv"),
           Scheme("uint4_asym", "group", 128, "fp16"), Scheme("int8_sym", "row")]
ROWS, COLS, N = 192, 4096, 5
SUM_RTOL = 1e-5


def _o(s: Scheme) -> oracle.Scheme:
    return oracle.Scheme(s.fmt, s.gran, s.block, s.scale_dtype, s.hadamard)


def _bytes(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.uint8).numpy().reshape(-1)


def _close(a, b, rtol=SUM_RTOL, atol=1e-30):
    return abs(a - b) <= atol + rtol * max(abs(a), abs(b))


def _gains(i: int) -> tuple[float, float]:
    # every call sees a different input: a power-of-two gain and an offset
    return float(2.0 ** (i - 2)), 0.125 * i


def _expected(s: Scheme, x: torch.Tensor):
    o = oracle.quantize(synth.bf16_bits(x.cpu()), _o(s))
    oxh = oracle.dequantize(o["codes"], o["scales"], o["zps"], o["tensor_scale"], ROWS, COLS, _o(s))
    return o, oxh


def _check_deq(oxh: np.ndarray, deq: torch.Tensor, what: str):
    assert np.array_equal(deq.cpu().numpy().view(np.uint32), oxh.view(np.uint32)), f"{what}: dequantized values"


def _check(s: Scheme, x: torch.Tensor, codes, scales, stats, deq: torch.Tensor, what: str):
    o, oxh = _expected(s, x)
    assert np.array_equal(codes.cpu().numpy(), o["codes"]), f"{what}: codes"
    assert np.array_equal(_bytes(scales), np.ascontiguousarray(o["scales"]).view(np.uint8).reshape(-1)), f"{what}: scales"
    _check_deq(oxh, deq, what)
    st, ost = stats.cpu().numpy(), o["stats"]
    assert _close(st[1], ost[1]) and _close(st[0], ost[0], atol=1e-30 + 1e-7 * ost[1]), (what, st, ost)
    assert st[4] == ost[4], (what, st, ost)


@pytest.mark.parametrize("s", SCHEMES, ids=str)
def test_producer_kernel_then_quantize_then_dequantize(s, cuda_device):
    """Read after write: a torch kernel writes each input right before its quantize, the
    dequantize reads the codes right after, and one workspace serves every call."""
    base = synth.weight_outliers(ROWS, COLS, seed=31).to(cuda_device)
    ws = bq.new_workspace(cuda_device)
    st = torch.cuda.Stream(cuda_device)
    st.wait_stream(torch.cuda.current_stream(cuda_device))
    res = []
    with torch.cuda.stream(st):
        for i in range(N):
            g, c = _gains(i)
            x = (base.float() * g + c).to(torch.bfloat16)
            q = bq.quantize(x, s, stats=True, workspace=ws)
            d = bq.dequantize(q, torch.float32)
            res.append((x, q, d))
    st.synchronize()
    for i, (x, q, d) in enumerate(res):
        _check(s, x, q.codes, q.scales, q.stats, d, f"{s} call {i}")


@pytest.mark.parametrize("s", SCHEMES, ids=str)
def test_quantize_overwrites_what_the_dequantize_ahead_reads(s, cuda_device):
    """Write after read: every quantize writes the same code, scale and stats buffers that
    the dequantize launched just before it is reading; each dequantized result must be
    that of its own input."""
    base = synth.activations_t3(ROWS, COLS, seed=32, n_outlier_channels=3).to(cuda_device)
    ws = bq.new_workspace(cuda_device)
    xs = [(base.float() * _gains(i)[0] + _gains(i)[1]).to(torch.bfloat16) for i in range(N)]
    q = bq.alloc_outputs(s.resolved(), ROWS, COLS, cuda_device)
    deqs = [torch.empty((ROWS, COLS), dtype=torch.float32, device=cuda_device) for _ in range(N)]
    st = torch.cuda.Stream(cuda_device)
    st.wait_stream(torch.cuda.current_stream(cuda_device))
    with torch.cuda.stream(st):
        for i in range(N):
            bq.quantize(xs[i], s, stats=True, workspace=ws, out=q)
            bq.dequantize(q, torch.float32, out=deqs[i])
    st.synchronize()
    for i in range(N - 1):
        _check_deq(_expected(s, xs[i])[1], deqs[i], f"{s} call {i}")
    _check(s, xs[N - 1], q.codes, q.scales, q.stats, deqs[N - 1], f"{s} call {N - 1}")


@pytest.mark.parametrize("s", [Scheme("int8_sym", "mx"), Scheme("e4m3", "tensor"), Scheme("e2m1", "nv")], ids=str)
def test_chain_inside_a_cuda_graph(s, cuda_device):
    """The same chains captured into one CUDA graph (the launches become graph nodes with
    programmatic edges), replayed twice."""
    base = synth.weight_outliers(ROWS, COLS, seed=33).to(cuda_device)
    ws = bq.new_workspace(cuda_device)
    sr = s.resolved()
    xs = [torch.empty((ROWS, COLS), dtype=torch.bfloat16, device=cuda_device) for _ in range(N)]
    qs = [bq.alloc_outputs(sr, ROWS, COLS, cuda_device) for _ in range(N)]
    deqs = [torch.empty((ROWS, COLS), dtype=torch.float32, device=cuda_device) for _ in range(N)]
    qsnrs = [torch.empty(5, dtype=torch.float64, device=cuda_device) for _ in range(N)]

    def chain(stream):
        for i in range(N):
            g, c = _gains(i)
            xs[i].copy_(base.float() * g + c)
            bq.bq_quantize(xs[i], sr, qs[i].codes, qs[i].scales, qs[i].zero_points, qs[i].tensor_scale,
                           qs[i].stats, ws, stream)
            bq.bq_dequantize(qs[i].codes, qs[i].scales, qs[i].zero_points, qs[i].tensor_scale, ROWS, COLS, sr,
                             deqs[i], stream)
            bq.bq_qsnr(xs[i], qs[i].codes, qs[i].scales, qs[i].zero_points, qs[i].tensor_scale, sr, qsnrs[i], ws,
                       stream)

    cap = torch.cuda.Stream(cuda_device)
    cap.wait_stream(torch.cuda.current_stream(cuda_device))
    with torch.cuda.stream(cap):
        chain(cap)                                   # eager once (the library's first launches)
    cap.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=cap):
        chain(cap)
    for _ in range(2):
        for t in deqs + qsnrs:
            t.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize(cuda_device)
        for i in range(N):
            _check(s, xs[i], qs[i].codes, qs[i].scales, qs[i].stats, deqs[i], f"{s} graph call {i}")
            xb = synth.bf16_bits(xs[i].cpu())
            o = oracle.quantize(xb, _o(s), stats=False)
            oq = oracle.qsnr_sums(xb, o["codes"], o["scales"], o["zps"], o["tensor_scale"], _o(s))
            qv = qsnrs[i].cpu().numpy()
            assert _close(qv[1], oq[1]) and _close(qv[0], oq[0], atol=1e-30 + 1e-7 * oq[1]), (i, qv, oq)
    del graph
