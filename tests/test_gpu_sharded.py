"""One tensor split by rows across two ranks (block_scaled_bit_bq_b200.sharded): the ranks'
concatenated codes and scales equal the oracle's for the whole tensor, and the combined
QSNR / kappa sums match the oracle's whole-tensor sums.

The two ranks are processes with a gloo group (the collectives run on host copies),
both on cuda:0: each rank's kernels run on its own data and never wait on the other
rank's; only the host-side all-reduces connect them.
"""

import datetime
import math
import multiprocessing as mp
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
pytestmark = pytest.mark.gpu

SCHEMES = [("e4m3", "tensor", 0, "fp32", False), ("int8_asym", "tensor", 0, "fp32", False),
           ("e2m1", "nv", 16, "e4m3", False), ("int4_sym", "nv", 16, "e4m3", True),
           ("int8_sym", "mx", 32, "ue8m0", False)]
ROWS, COLS, SPLIT = 300, 1024, 137


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, port, out):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch
    import torch.distributed as dist
    import synth
    from block_scaled_bit_bq_b200 import Scheme, sharded
    dist.init_process_group("gloo", rank=rank, world_size=2, timeout=datetime.timedelta(seconds=60))
    try:
        x = synth.activations_t3(ROWS, COLS, seed=901, n_outlier_channels=2)
        lo, hi = (0, SPLIT) if rank == 0 else (SPLIT, ROWS)
        xd = x[lo:hi].to("cuda:0")
        res = []
        for a in SCHEMES:
            q, st = sharded.quantize_rows_shard(xd, Scheme(*a), ROWS)
            res.append((q.codes.cpu().numpy(), q.scales.cpu().view(torch.uint8).numpy(),
                        None if q.zero_points is None else q.zero_points.cpu().view(torch.uint8).numpy(),
                        None if q.tensor_scale is None else q.tensor_scale.cpu().numpy(), st.cpu().numpy()))
        out.put((rank, res))
    finally:
        dist.destroy_process_group()


def test_two_ranks_quantize_one_tensor(cuda_device):
    import oracle
    import synth
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    xb = synth.bf16_bits(synth.activations_t3(ROWS, COLS, seed=901, n_outlier_channels=2))
    for i, a in enumerate(SCHEMES):
        o = oracle.quantize(xb, oracle.Scheme(*a))
        c0, s0, z0, t0, st0 = got[0][i]
        c1, s1, z1, t1, st1 = got[1][i]
        assert np.array_equal(np.concatenate([c0, c1]), o["codes"]), a
        osc = o["scales"].view(np.uint8).reshape(-1)
        if a[1] == "tensor":
            assert np.array_equal(s0, osc) and np.array_equal(s1, osc), a
            if o["zps"] is not None:
                oz = o["zps"].view(np.uint8).reshape(-1)
                assert np.array_equal(z0, oz) and np.array_equal(z1, oz), a
        else:
            assert np.array_equal(np.concatenate([s0, s1]), osc), a
        if o["tensor_scale"] is not None:
            assert t0[0] == o["tensor_scale"][0] and t1[0] == o["tensor_scale"][0], a
        ost = o["stats"]
        for st in (st0, st1):                         # every rank holds the whole tensor's sums
            assert abs(st[0] - ost[0]) <= 1e-5 * ost[0] + 1e-7 * ost[1] and abs(st[1] - ost[1]) <= 1e-5 * ost[1], a
            assert abs(-10 * math.log10(st[0] / st[1]) - oracle.qsnr_db(ost[0], ost[1])) < 0.01, a
            assert st[4] == ost[4] and abs(st[2] - ost[2]) <= 1e-5 * ost[2] and abs(st[3] - ost[3]) <= 1e-5 * ost[3], a
