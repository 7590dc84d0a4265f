"""GPU parity: the CUDA library against the CPU oracle, through the C ABI.

Codes, scales, zero points, tensor scales and dequantized values (fp32 and bf16) must
match bit for bit; QSNR within 0.01 dB; the sums behind it and the crest-factor sums
within 1e-5 relative (fp32 partial sums on the GPU, double on the CPU).
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

QSNR_TOL_DB = 0.01
SUM_RTOL = 1e-5

ALL_SCHEMES = [
    Scheme("int8_sym", "tensor"), Scheme("int8_sym", "tensor", scale_dtype="fp16"),
    Scheme("int8_sym", "row"), Scheme("int8_sym", "group", 64), Scheme("int8_sym", "group", 16),
    Scheme("int8_sym", "group", 512, "fp16"),
    Scheme("int8_asym", "tensor"), Scheme("int8_asym", "row", scale_dtype="fp16"),
    Scheme("int8_asym", "group", 128, "fp16"), Scheme("int8_asym", "group", 32),
    Scheme("int4_sym", "tensor"), Scheme("int4_sym", "row"), Scheme("int4_sym", "group", 64),
    Scheme("int4_sym", "group", 256, "fp16"),
    Scheme("uint4_asym", "tensor", scale_dtype="fp16"), Scheme("uint4_asym", "row"),
    Scheme("uint4_asym", "group", 128, "fp16"), Scheme("uint4_asym", "group", 64),
    Scheme("e4m3", "tensor"), Scheme("e4m3", "row"), Scheme("e4m3", "group", 128),
    Scheme("e4m3", "row", scale_dtype="fp16"),
    Scheme("e5m2", "tensor"), Scheme("e5m2", "row"), Scheme("e5m2", "group", 32, "fp16"),
    Scheme("int8_sym", "mx"), Scheme("e4m3", "mx"), Scheme("e5m2", "mx"), Scheme("e2m1", "mx"),
    Scheme("e2m1", "nv"), Scheme("int4_sym", "nv"),
    Scheme("int4_sym", "nv", hadamard=True), Scheme("e2m1", "nv", hadamard=True),
    Scheme("int8_sym", "row", hadamard=True), Scheme("e4m3", "tensor", hadamard=True),
    Scheme("uint4_asym", "group", 128, "fp16", hadamard=True), Scheme("int8_sym", "mx", hadamard=True),
    Scheme("e2m3", "mx"), Scheme("e3m2", "mx"), Scheme("e2m3", "mx", hadamard=True),
    Scheme("int8_sym", "tile2d"), Scheme("int8_asym", "tile2d", scale_dtype="fp16"),
    Scheme("int4_sym", "tile2d", scale_dtype="fp16"), Scheme("uint4_asym", "tile2d"),
    Scheme("e4m3", "tile2d"), Scheme("e5m2", "tile2d", scale_dtype="fp16"),
    Scheme("e4m3", "tile2d", hadamard=True), Scheme("uint4_asym", "tile2d", scale_dtype="fp16", hadamard=True),
]


def _o(s: Scheme) -> oracle.Scheme:
    return oracle.Scheme(s.fmt, s.gran, s.block, s.scale_dtype, s.hadamard)


def _bytes(a) -> np.ndarray:
    if isinstance(a, torch.Tensor):
        a = a.detach().cpu().contiguous()
        return a.view(torch.uint8).numpy().reshape(-1)
    return np.ascontiguousarray(a).view(np.uint8).reshape(-1)


def _close(a, b, rtol=SUM_RTOL, atol=1e-30):
    if math.isinf(a) or math.isinf(b):
        return a == b        # e.g. MX codes near the bf16 maximum dequantize past fp32
    return abs(a - b) <= atol + rtol * max(abs(a), abs(b))


def check(x: torch.Tensor, s: Scheme, ws: torch.Tensor, what: str = "", full_stats: bool = True,
          tensor_range=None, rows_sample=None):
    """Quantize x (CPU bf16 [rows, cols]) on both sides and compare everything."""
    rows, cols = x.shape
    xb = synth.bf16_bits(x)
    xd = x.cuda()
    q = bq.quantize(xd, s, stats=True, workspace=ws)
    deq32 = bq.dequantize(q, torch.float32)
    deq16 = bq.dequantize(q, torch.bfloat16)
    qs = bq.qsnr(xd, q, workspace=ws)
    torch.cuda.synchronize()

    if rows_sample is None:
        o = oracle.quantize(xb, _o(s))
        sel = slice(None)
    else:
        # rows drawn from a full-size tensor: per-tensor quantities come from the whole
        sel = np.asarray(rows_sample)
        o = oracle.quantize(xb[sel], _o(s), tensor_range=tensor_range, stats=False)
    oxh = oracle.dequantize(o["codes"], o["scales"], o["zps"], o["tensor_scale"], o["codes"].shape[0], cols, _o(s))

    codes = q.codes.cpu().numpy()[sel]
    assert np.array_equal(codes, o["codes"]), f"{what} {s}: codes differ at {np.argwhere(codes != o['codes'])[:5]}"
    if rows_sample is None or s.gran in ("tensor",):
        sc_gpu, sc_or = _bytes(q.scales), _bytes(o["scales"])
        if rows_sample is not None:
            sc_gpu = sc_gpu[:sc_or.size]
        assert np.array_equal(sc_gpu, sc_or), f"{what} {s}: scales differ"
    else:
        per_row = q.scales.numel() // rows
        g = q.scales.cpu().reshape(rows, per_row)[torch.as_tensor(sel)]
        assert np.array_equal(_bytes(g), _bytes(o["scales"])), f"{what} {s}: scales differ"
    if o["zps"] is not None:
        if rows_sample is None or s.gran == "tensor":
            assert np.array_equal(_bytes(q.zero_points)[:_bytes(o["zps"]).size], _bytes(o["zps"])), f"{what} {s}: zps"
        else:
            per_row = q.zero_points.numel() // rows
            g = q.zero_points.cpu().reshape(rows, per_row)[torch.as_tensor(sel)]
            assert np.array_equal(_bytes(g), _bytes(o["zps"])), f"{what} {s}: zero points differ"
    if o["tensor_scale"] is not None:
        assert np.array_equal(_bytes(q.tensor_scale), _bytes(o["tensor_scale"])), f"{what} {s}: tensor scale"

    d32 = deq32.cpu().numpy()[sel]
    bad = np.nonzero(d32.view(np.uint32) != oxh.view(np.uint32))
    assert bad[0].size == 0, f"{what} {s}: fp32 dequant differs at {list(zip(*bad))[:5]}"
    d16 = _bytes(deq16.cpu()[torch.as_tensor(sel)] if rows_sample is not None else deq16).view(np.uint16)
    assert np.array_equal(d16, oracle.to_bf16_array(oxh).reshape(-1)), f"{what} {s}: bf16 dequant differs"

    if full_stats and rows_sample is None:
        st = q.stats.cpu().numpy()
        ost = o["stats"]
        assert _close(st[1], ost[1]), (what, s, st, ost)
        assert _close(st[0], ost[0], atol=1e-30 + 1e-7 * ost[1]), (what, s, st, ost)
        if ost[0] > 0 and ost[1] > 0 and math.isfinite(ost[0]):
            assert abs(bq.bq_stats_qsnr_db(st) - oracle.qsnr_db(ost[0], ost[1])) < QSNR_TOL_DB
        assert st[4] == ost[4], (what, s, st, ost)
        assert _close(st[2], ost[2]) and _close(st[3], ost[3]), (what, s, st, ost)
        qv = qs.cpu().numpy()
        oq = oracle.qsnr_sums(xb, o["codes"], o["scales"], o["zps"], o["tensor_scale"], _o(s))
        assert _close(qv[1], oq[1]) and _close(qv[0], oq[0], atol=1e-30 + 1e-7 * oq[1]), (what, s, qv, oq)
        assert qv[2] == 0 and qv[3] == 0 and qv[4] == 0
    return q


@pytest.fixture(scope="module")
def ws(cuda_device):
    return bq.new_workspace(cuda_device)


def _valid(s: Scheme, cols: int) -> bool:
    try:
        oracle.buffer_sizes(_o(s), 1, cols)
        return True
    except ValueError:
        return False


def _edge_tensor(rows=8, cols=512, seed=5, big=1.5e38):
    g = np.random.default_rng(seed)
    a = (g.standard_t(3, size=(rows, cols)) * 0.5).astype(np.float32)
    a[0] = 0.0                                                   # all-zero row
    a[1] = (g.standard_normal(cols) * 1e-39).astype(np.float32)   # bf16 subnormals
    a[2] = (g.uniform(-1, 1, cols) * big).astype(np.float32)      # huge values of both signs
    a[6] = (g.uniform(0.5, 1, cols) * 2.2 * big).astype(np.float32)   # up to the bf16 maximum
    # ties: multiples of 1/2 and 1/4 of a power of two under a power-of-two amax
    a[3] = (g.integers(-64, 65, cols) * 0.5).astype(np.float32)
    a[3, 0] = 64.0
    a[4] = -0.0
    a[4, ::3] = (g.integers(-8, 9, (cols + 2) // 3) * 0.25).astype(np.float32)
    a[5, :] = 1.0                                                # constant row
    return synth.to_bf16(a)


INPUTS = {
    "weight_37x1024": lambda: synth.weight_outliers(37, 1024, seed=101),
    "t3_16x4096": lambda: synth.activations_t3(16, 4096, seed=102, n_outlier_channels=3),
    "edge_8x512": lambda: _edge_tensor(),
    # rotated schemes take |x| <= 2^125
    "edge_rot_8x512": lambda: _edge_tensor(big=1.5e38 / 16),
    "ragged_5x48": lambda: synth.normal(5, 48, seed=103, sigma=3.0),
    # 129 and 387 chunks: the last warp tile holds only the ragged end (no whole row)
    "tail_1x2064": lambda: synth.normal(1, 2064, seed=106, sigma=2.0),
    "tail_3x2064": lambda: synth.weight_outliers(3, 2064, seed=107),
    "single_1x16": lambda: synth.uniform(1, 16, seed=104),
    "uniform_3x2048": lambda: synth.uniform(3, 2048, seed=105),
    # three 128-row tile rows, the last of 44 rows; three tile columns
    "tiles_300x384": lambda: synth.weight_outliers(300, 384, seed=108),
}


@pytest.mark.parametrize("name", list(INPUTS))
@pytest.mark.parametrize("s", ALL_SCHEMES, ids=str)
def test_parity_small(s, name, ws):
    x = INPUTS[name]()
    if not _valid(s, x.shape[1]):
        pytest.skip("scheme does not divide this shape")
    if s.hadamard and name == "edge_8x512":
        pytest.skip("rotated schemes take |x| <= 2^125 (see edge_rot_8x512)")
    check(x, s, ws, name)


@pytest.mark.parametrize("cols", [16, 96, 640, 2112, 3136, 4096, 4160, 6144, 8192, 12288, 16384, 20480])
@pytest.mark.parametrize("s", [Scheme("int8_sym", "row"), Scheme("uint4_asym", "row", scale_dtype="fp16"),
                               Scheme("e5m2", "row", hadamard=True)], ids=str)
def test_row_kernel_shapes(s, cols, ws):
    # cols % 64 != 0 (16, 96): a CTA per row; other widths: a warp per row through the
    # segment tensor map, with a partly filled last tile (640, 2112, 3136, 4160) or whole tiles;
    # rows of 3-4 tiles (4160, 6144, 8192) take the four-stage ring
    x = synth.activations_t3(9, cols, seed=200 + cols, n_outlier_channels=1)
    check(x, s, ws, f"rows9x{cols}")


@pytest.mark.parametrize("s", [Scheme("int8_sym", "row"), Scheme("e4m3", "row")], ids=str)
def test_row_kernel_rows_through_the_ring(s, ws):
    # more rows than warps: each warp takes several 6144-column rows (three tiles) through
    # the four-stage ring that keeps a row resident for both passes
    x = synth.activations_t3(2000, 6144, seed=260, n_outlier_channels=2)
    check(x, s, ws, "rows2000x6144")


@pytest.mark.parametrize("rows", [1, 127, 128, 129, 640])
@pytest.mark.parametrize("s", [Scheme("e4m3", "tile2d"), Scheme("uint4_asym", "tile2d", scale_dtype="fp16")], ids=str)
def test_tile2d_shapes(s, rows, ws):
    # tile rows of 1..128 rows, whole and ragged, over more tiles than one wave of CTAs
    # at 640 x 8192 (320 tiles)
    cols = 8192 if rows == 640 else 1152
    x = synth.weight_outliers(rows, cols, seed=300 + rows)
    check(x, s, ws, f"tiles{rows}x{cols}")


def test_empty_input(ws, cuda_device):
    for s in [Scheme("int8_sym", "tensor"), Scheme("e2m1", "nv"), Scheme("int8_sym", "row"), Scheme("e4m3", "tile2d")]:
        x = torch.empty((0, 128), dtype=torch.bfloat16, device=cuda_device)
        st = torch.full((5,), 7.0, dtype=torch.float64, device=cuda_device)
        q = bq.alloc_outputs(s, 0, 128, cuda_device)
        codes = torch.empty(0, dtype=torch.uint8, device=cuda_device)
        bq.bq_quantize(x, s, codes, q.scales, q.zero_points, q.tensor_scale, st, ws)
        torch.cuda.synchronize()
        assert st.cpu().tolist() == [0.0] * 5


def test_stats_are_deterministic(ws):
    x = synth.weight_outliers(512, 4096, seed=7).cuda()
    for s in [Scheme("uint4_asym", "group", 128, "fp16"), Scheme("e4m3", "tensor"), Scheme("int8_sym", "row")]:
        a = bq.quantize(x, s, workspace=ws).stats.cpu()
        b = bq.quantize(x, s, workspace=ws).stats.cpu()
        assert torch.equal(a, b)


def test_side_stream(ws):
    x = synth.weight_outliers(64, 1024, seed=9).cuda()
    s = Scheme("e4m3", "tensor")
    st = torch.cuda.Stream()
    ref = bq.quantize(x, s, workspace=ws)
    torch.cuda.synchronize()
    with torch.cuda.stream(st):
        q = bq.quantize(x, s, workspace=ws, stream=st)
    st.synchronize()
    assert torch.equal(q.codes, ref.codes) and torch.equal(q.scales, ref.scales)


# ---------------------------------------------------------------------------
# the five workloads at full size
# ---------------------------------------------------------------------------

def test_tiny_weight_full(ws):
    x = synth.tiny_weight()
    for s in [Scheme("int8_sym", "tensor"), Scheme("int4_sym", "group", 64)]:
        check(x, s, ws, "tiny_weight")


def test_weight_outliers_full(ws):
    x = synth.weight_outliers()
    for s in [Scheme("uint4_asym", "group", 128, "fp16"), Scheme("int8_sym", "row"),
              Scheme("e4m3", "tile2d"), Scheme("e4m3", "group", 128)]:
        check(x, s, ws, "weight_outliers")


def test_activations_t3_full(ws):
    x = synth.activations_t3()
    for s in [Scheme("e4m3", "tensor"), Scheme("e5m2", "tensor"), Scheme("e4m3", "row"), Scheme("e5m2", "row")]:
        check(x, s, ws, "activations_t3")


@pytest.mark.parametrize("t", [0, 63])
def test_ffn_lognormal_full(t, ws):
    x = synth.ffn_lognormal(t)
    for s in [Scheme("int8_sym", "mx"), Scheme("e4m3", "mx")]:
        check(x, s, ws, f"ffn_lognormal[{t}]")


def test_weight_x50_full(ws):
    # every row of the 8192 x 28672 tensor: codes, block scales, the tensor scale, the fp32
    # and bf16 dequantized values, the fused and standalone QSNR sums and the kappa sums
    x = synth.weight_x50()
    for s in [Scheme("e2m1", "nv"), Scheme("int4_sym", "nv"), Scheme("int4_sym", "nv", hadamard=True)]:
        check(x, s, ws, "weight_x50")


RANGE_SCHEMES = [Scheme("int8_sym", "tensor"), Scheme("int8_asym", "tensor"), Scheme("uint4_asym", "tensor", scale_dtype="fp16"),
                 Scheme("e4m3", "tensor"), Scheme("e5m2", "tensor", hadamard=True), Scheme("e2m1", "nv"),
                 Scheme("int4_sym", "nv", hadamard=True)]


@pytest.mark.parametrize("s", RANGE_SCHEMES, ids=str)
def test_range_split(s, ws, cuda_device):
    """bq_tensor_range then bq_quantize_with_range gives bq_quantize's results; a row block
    quantized against the whole tensor's range gives the oracle's codes for those rows."""
    x = synth.activations_t3(300, 1024, seed=400, n_outlier_channels=2)
    xb = synth.bf16_bits(x)
    xd = x.to(cuda_device)
    rng = torch.empty(3, dtype=torch.float32, device=cuda_device)
    bq.bq_tensor_range(xd, s, rng, ws)
    ref = bq.quantize(xd, s, workspace=ws)
    q = bq.alloc_outputs(s, 300, 1024, cuda_device)
    bq.bq_quantize_with_range(xd, s, rng, q.codes, q.scales, q.zero_points, q.tensor_scale, q.stats, ws)
    torch.cuda.synchronize()
    tr = oracle.tensor_range(xb, s.hadamard)
    r = rng.cpu().numpy()
    asym_tensor = s.fmt in ("int8_asym", "uint4_asym") and s.gran == "tensor"
    want = np.array([tr[0], min(tr[1], 0.0) if asym_tensor else 0.0, max(tr[2], 0.0) if asym_tensor else 0.0],
                    dtype=np.float32)
    assert np.array_equal(r.view(np.uint32), want.view(np.uint32)), (r, tr)
    for a, b in [(q.codes, ref.codes), (q.scales, ref.scales), (q.zero_points, ref.zero_points),
                 (q.tensor_scale, ref.tensor_scale), (q.stats, ref.stats)]:
        if a is not None:
            assert torch.equal(a.view(torch.uint8), b.view(torch.uint8)), s
    # rows 100..227 of the tensor under the whole tensor's range (one shard of a split tensor)
    part = xd[100:228].contiguous()
    qp = bq.alloc_outputs(s, 128, 1024, cuda_device)
    bq.bq_quantize_with_range(part, s, rng, qp.codes, qp.scales, qp.zero_points, qp.tensor_scale, None, None)
    torch.cuda.synchronize()
    o = oracle.quantize(xb[100:228], _o(s), tensor_range=tr, stats=False)
    assert np.array_equal(qp.codes.cpu().numpy(), o["codes"]), s
    assert np.array_equal(_bytes(qp.scales), _bytes(o["scales"])), s
    if o["tensor_scale"] is not None:
        assert np.array_equal(_bytes(qp.tensor_scale), _bytes(o["tensor_scale"])), s


def test_no_tile_wait_gave_up(cuda_device):
    # every staged tile of every call above arrived (bounded waits never ran out)
    assert bq.bq_wait_timeouts() == 0


@pytest.mark.parametrize("s", [Scheme("e4m3", "tensor"), Scheme("e4m3", "row"), Scheme("e5m2", "group", 128),
                               Scheme("e4m3", "group", 32, "fp16"), Scheme("e2m1", "nv"), Scheme("e4m3", "mx"),
                               Scheme("e2m1", "mx")], ids=str)
def test_negative_zero_keeps_its_sign(s, ws):
    # a tensor of one row: -0.0 and tiny negatives next to ordinary values, alone in its
    # warp, so the fast FP path (not the general one) codes it; the oracle keeps the sign
    # of a zero result (codes 0x80 / 0x8)
    a = np.full((1, 512), -0.0, dtype=np.float32)
    a[0, ::4] = np.linspace(-2.0, 2.0, 128, dtype=np.float32)
    a[0, 1::16] = -1e-30
    check(synth.to_bf16(a), s, ws, "negative zeros")
