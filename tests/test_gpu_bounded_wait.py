"""The quantize kernels' bounded tile waits, made to run out without faulting the GPU.

bq_debug_skip_tile_copy makes the next flat quantize launch skip the copy of one staged
tile, so the mbarrier that warp waits on is never completed: a flag that nothing sets.
The wait gives up after its one-second limit, the warp waits (bounded) for its other
copies in flight and stops, and bq_wait_timeouts counts it. Nothing is left in flight
when the kernel ends. The next call on the same workspace must be exact again.
"""

import time

import numpy as np
import pytest
import torch

import oracle
import synth
import block_scaled_bit_bq_b200 as bq
from block_scaled_bit_bq_b200 import Scheme

pytestmark = pytest.mark.gpu


def test_wait_runs_out_and_the_next_call_is_exact(cuda_device):
    ws = bq.new_workspace(cuda_device)
    s = Scheme("int8_sym", "group", 64)
    x = synth.weight_outliers(64, 1024, seed=31)       # 4096 chunks: 32 staged tiles
    xb = synth.bf16_bits(x)
    xd = x.to(cuda_device)
    bq.bq_wait_timeouts(reset=True)
    q = bq.alloc_outputs(s, 64, 1024, cuda_device)
    bq.bq_debug_skip_tile_copy(0)
    t0 = time.time()
    bq.bq_quantize(xd, s, q.codes, q.scales, q.zero_points, q.tensor_scale, q.stats, ws)
    torch.cuda.synchronize()
    dt = time.time() - t0
    # the first wait and the drain of the skipped stage each run out after about a second
    assert 1.0 <= dt < 20.0, dt
    assert bq.bq_wait_timeouts() == 1
    # the hook is one-shot: the next call runs normally on the same workspace
    q2 = bq.quantize(xd, s, workspace=ws)
    torch.cuda.synchronize()
    o = oracle.quantize(xb, oracle.Scheme("int8_sym", "group", 64, "fp32", False))
    assert np.array_equal(q2.codes.cpu().numpy(), o["codes"])
    assert np.array_equal(q2.scales.cpu().numpy().view(np.uint32), o["scales"].view(np.uint32))
    st = q2.stats.cpu().numpy()
    assert abs(bq.bq_stats_qsnr_db(st) - oracle.qsnr_db(o["stats"][0], o["stats"][1])) < 0.01
    assert st[4] == o["stats"][4]
    assert bq.bq_wait_timeouts() == 1
    bq.bq_wait_timeouts(reset=True)
    assert bq.bq_wait_timeouts() == 0
