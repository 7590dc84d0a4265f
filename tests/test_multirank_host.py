"""The multi-GPU host logic of bench.py on CPU: two gloo ranks (no GPU).

Each rank owns an independent tensor (weak scaling, no collective on the data path);
the harness takes the max of the per-rank step times and reports the whole-job
throughput from it.
"""

import datetime
import multiprocessing as mp
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        ms = 1.0 + 0.5 * rank                     # this rank's step time
        m = bench.reduce_max(ms)
        bench.barrier()
        x = bench.gen_inputs("tiny_weight", rank, 1)[0]
        out.put((rank, m, bench.aggregate(1.0e9, world, m), float(x.float().abs().sum())))
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_max_time_and_own_distinct_tensors():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, m0, v0, s0), (r1, m1, v1, s1) = res
    assert m0 == m1 == 1.5                        # max over ranks
    assert v0 == v1 == pytest.approx(2 * 1.0e9 / 1.5e-3 / 1e9)
    assert s0 != s1                               # independent inputs per rank


def test_single_process_helpers():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max(3.0) == 3.0          # no process group: identity
    kb = bench.kernel_bytes((1 << 20, 4096, 0, 0), 1024, 2048)
    assert kb["quantize"] == kb["quantize_pass"] == 2 * 1024 * 2048 + (1 << 20) + 4096
    assert kb["dequantize"] == (1 << 20) + 4096 + 2 * 1024 * 2048
    assert kb["range"] == 2 * 1024 * 2048
    a = bench.gen_inputs("tiny_weight", 0, 1)[0]
    b = bench.gen_inputs("tiny_weight", 0, 1)[0]
    import torch
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))   # same seed, same bytes
    # the FFN set: rank r owns tensors 64 r .. 64 r + 63 (seed 3 + t); rank 0 owns the
    # 64 tensors of the workload, drawn in parallel but identical to one-by-one draws
    import synth
    f = bench.gen_inputs("ffn_lognormal", 0, 3)
    assert len(f) == 3 and torch.equal(f[2].view(torch.int16), synth.ffn_lognormal(2).view(torch.int16))
    g = bench.gen_inputs("ffn_lognormal", 1, 3)
    assert torch.equal(g[0].view(torch.int16), synth.ffn_lognormal(3).view(torch.int16))
    assert [(a, b) for a, b in bench._blocks(10, 4)] == [(0, 2), (2, 5), (5, 7), (7, 10)]
    assert bench._blocks(2, 8) == [(0, 1), (1, 2)]


def test_bench_oracle_arm_covers_every_workload():
    # every bench workload's schemes are valid oracle schemes, and the oracle step (the
    # cpu_baseline leg and the reference arm) runs on a few rows of each, with the
    # rotation where the workload asks for it
    sys.path.insert(0, ROOT)
    import bench
    import synth
    for w, schemes in bench.WORKLOADS.items():
        rows = 2
        cols = {"tiny_weight": 1024}.get(w, 4096)
        x = synth.bf16_bits(synth.normal(rows, cols, seed=5, sigma=0.02))
        signs = bench.rotation_signs(w, cols)
        bench.oracle_step(x, schemes, signs)
        bench.oracle_step(x, schemes, signs, threads=2)        # row blocks on two threads
        assert bench.oracle_bytes(schemes, rows, cols) > 2 * rows * cols * len(schemes)
    assert bench.rotation_signs("weight_outliers", 4096) is None
    s = bench.rotation_signs("weight_rotated", 4096)
    assert s.shape == (4096,) and set(np.unique(s)) <= {0, 1}


def test_reference_arm_prints_the_contract_line():
    # bench.py --impl reference: the oracle timed on this host, one JSON line with the
    # contract's keys (no GPU needed)
    import json
    import subprocess
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                        "tiny_weight", "--steps", "3", "--warmup", "3", "--cpu-seconds", "1"],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    d = json.loads(r.stdout.strip().splitlines()[-1])
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["value"] > 0
    assert d["higher_is_better"] is True and d["steps"] == 3 and d["warmup"] == 3
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] == bench_cores()
    assert d["cpu_baseline"]["value"] == d["value"] and "rows" in d["cpu_baseline"]["sample"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["config"]["workload"].startswith("tiny_weight: bf16 256x1024")


def bench_cores():
    sys.path.insert(0, ROOT)
    import bench
    return bench.host_cores()


def _combine_worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        from block_scaled_bit_bq_b200 import sharded
        # rank 0's block: amax 3, min -3, max 1; rank 1's: amax 5, min 0, max 5
        local = torch.tensor([[3.0, -3.0, 1.0], [5.0, 0.0, 5.0]][rank])
        rng = sharded.combine_ranges(local)
        st = torch.tensor([[1.0, 10.0, 2.0, 1.5, 4.0], [3.0, 30.0, 6.0, 2.5, 8.0]][rank], dtype=torch.float64)
        blocks = sharded.combine_stats(st, None, 100)
        tensor = sharded.combine_stats(st, 5.0, 100)
        out.put((rank, rng.tolist(), blocks.tolist(), tensor.tolist()))
    finally:
        dist.destroy_process_group()


def test_two_ranks_combine_ranges_and_stats():
    # the split-tensor path's two collectives: ranges (MAX of amax and max, MIN of min) and
    # stats (sums added, kappa max taken; a per-tensor scheme's one kappa from the totals)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_combine_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, rng, blocks, tensor in res:
        assert rng == [5.0, -3.0, 5.0]
        assert blocks == [4.0, 40.0, 8.0, 2.5, 12.0]
        k = 5.0 / (40.0 / 100) ** 0.5
        assert tensor[:2] == [4.0, 40.0] and abs(tensor[2] - k) < 1e-12 and tensor[3] == tensor[2] and tensor[4] == 1.0
