"""bq_quantize_noalloc: quantize with the library's static device scratch.

For callers that cannot allocate device memory (their memory belongs to another
allocator, or a cudaMalloc would synchronize a pipeline that must stay asynchronous):
the call must give the same codes, scales, zero points, tensor scale and QSNR sums as
bq_quantize with a caller workspace, on consecutive calls that reuse the shared array.
"""

import numpy as np
import pytest
import torch

import synth
import block_scaled_bit_bq_b200 as bq
from block_scaled_bit_bq_b200 import Scheme

pytestmark = pytest.mark.gpu

SCHEMES = [Scheme("e4m3", "tensor"), Scheme("uint4_asym", "group", 128, "fp16"), Scheme("e2m1", "nv", hadamard=True),
           Scheme("int8_sym", "row")]


def _same(a, b):
    if a is None:
        return b is None
    return torch.equal(a.view(torch.uint8), b.view(torch.uint8))


@pytest.mark.parametrize("s", SCHEMES, ids=str)
def test_noalloc_matches_workspace_call_twice(s, cuda_device):
    ws = bq.new_workspace(cuda_device)
    for call, seed in enumerate((31, 32)):          # two calls in a row on the shared array
        x = synth.weight_outliers(96, 2048, seed=seed).to(cuda_device)
        ref = bq.alloc_outputs(s, 96, 2048, cuda_device)
        got = bq.alloc_outputs(s, 96, 2048, cuda_device)
        bq.bq_quantize(x, s.resolved(), ref.codes, ref.scales, ref.zero_points, ref.tensor_scale, ref.stats, ws)
        bq.bq_quantize_noalloc(x, s.resolved(), got.codes, got.scales, got.zero_points, got.tensor_scale, got.stats)
        torch.cuda.synchronize(cuda_device)
        assert torch.equal(got.codes, ref.codes), (s, call)
        assert _same(got.scales, ref.scales) and _same(got.zero_points, ref.zero_points), (s, call)
        assert _same(got.tensor_scale, ref.tensor_scale), (s, call)
        a, b = got.stats.cpu().numpy(), ref.stats.cpu().numpy()
        assert np.allclose(a, b, rtol=1e-12, atol=0), (s, call, a, b)
        assert abs(bq.bq_stats_qsnr_db(a) - bq.bq_stats_qsnr_db(b)) < 0.01
