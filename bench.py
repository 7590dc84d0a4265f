"""Benchmark of the block-scaled quantization hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload weight_outliers|tiny_weight|activations_t3|ffn_lognormal|ffn_mx_family|ffn_mx_gemm_operands|weight_tiles_fp8|weight_rotated|weight_x50]

A step is one pass of the whole path over one synthetic tensor of the workload:
quantize (with fused QSNR and crest-factor sums) under each of the workload's schemes,
then dequantize each result to bf16. The default workload is the 4096 x 4096 weight
(N(0, 0.02^2) with 0.1% entries +-U(0.1, 0.2)) under UINT4 group-128 asymmetric
(fp16 scale + zero) and INT8 per-output-channel symmetric.

value: algorithmic bytes of every kernel of a step (bytes each kernel must read plus
bytes it must write) / step time, summed over ranks (weak scaling: each rank owns an
independent tensor), with inputs resident in HBM. Inputs rotate over enough buffer sets
that every step reads data last touched more than 4 x L2 ago.
e2e: the same bytes / step time when every step also copies its input from pinned host
memory and reads its quantized outputs and QSNR sums back.

Under torchrun (N > 1) each rank drives cuda:LOCAL_RANK; times are the max over ranks.
--impl reference times the CPU oracle (the reference implementation here) on rank 0.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "quantize GB/s (bytes in+out) and % of B200 HBM peak; QSNR dB matching oracle"
KERNEL_SOURCES = ("common.cuh", "quant_ops.cuh", "tma.cuh", "rot.cuh", "quant_flat.cu", "quant_row.cu", "dequant.cu")

# workload -> (generator kwargs, list of (label, scheme args))
WORKLOADS = {
    "weight_outliers": [("uint4_g128_asym", ("uint4_asym", "group", 128, "fp16", False)),
                        ("int8_row_sym", ("int8_sym", "row", 0, "fp32", False))],
    "tiny_weight": [("int8_tensor_sym", ("int8_sym", "tensor", 0, "fp32", False)),
                    ("int4_g64_sym", ("int4_sym", "group", 64, "fp32", False))],
    "activations_t3": [("e4m3_tensor", ("e4m3", "tensor", 0, "fp32", False)),
                       ("e5m2_tensor", ("e5m2", "tensor", 0, "fp32", False)),
                       ("e4m3_token", ("e4m3", "row", 0, "fp32", False)),
                       ("e5m2_token", ("e5m2", "row", 0, "fp32", False))],
    "ffn_lognormal": [("mxint8", ("int8_sym", "mx", 32, "ue8m0", False)),
                      ("mxfp8_e4m3", ("e4m3", "mx", 32, "ue8m0", False))],
    # the rest of the MX family on the same FFN tensor (MXFP4 and MXFP6)
    "ffn_mx_family": [("mxfp4", ("e2m1", "mx", 32, "ue8m0", False)),
                      ("mxfp6_e2m3", ("e2m3", "mx", 32, "ue8m0", False)),
                      ("mxfp6_e3m2", ("e3m2", "mx", 32, "ue8m0", False))],
    # the DeepSeek-V3 FP8 recipe on the 4096 x 4096 outlier weight: E4M3 with one fp32
    # scale per 128 x 128 tile (weights), and per 1 x 128 tile (the activation tiling)
    "weight_tiles_fp8": [("e4m3_tile128x128", ("e4m3", "tile2d", 128, "fp32", False)),
                         ("e4m3_tile1x128", ("e4m3", "group", 128, "fp32", False))],
    # GEMM operands: MXFP8 and MXFP4 of the FFN tensor with the block scales written in
    # the layout a block-scaled tensor-core GEMM reads (128 x 4 tiles)
    "ffn_mx_gemm_operands": [("mxfp8_e4m3_gemm", ("e4m3", "mx", 32, "ue8m0", False, "gemm")),
                             ("mxfp4_gemm", ("e2m1", "mx", 32, "ue8m0", False, "gemm"))],
    # QuaRot-style: the 4096 x 4096 outlier weight under a randomized full-row Hadamard
    # rotation (random signs, seed 21), then MXFP4 and INT4 group-128
    "weight_rotated": [("mxfp4_rot", ("e2m1", "mx", 32, "ue8m0", False)),
                       ("int4_g128_rot", ("int4_sym", "group", 128, "fp32", False))],
    "weight_x50": [("nvfp4", ("e2m1", "nv", 16, "e4m3", False)),
                   ("nvint4", ("int4_sym", "nv", 16, "e4m3", False)),
                   ("nvint4_hadamard", ("int4_sym", "nv", 16, "e4m3", True))],
}


# workloads whose schemes all run after the randomized full-row rotation: sign seed
ROTATED = {"weight_rotated": 21}


def rotation_signs(workload: str, cols: int):
    """The workload's per-column sign flags (uint8 0/1), or None."""
    return synth.random_signs(cols, ROTATED[workload]) if workload in ROTATED else None


def gen_input(workload: str, rank: int) -> torch.Tensor:
    """The rank's tensor: the workload's generator with its seed shifted by 1000 * rank."""
    if workload in ("ffn_lognormal", "ffn_mx_family", "ffn_mx_gemm_operands"):
        return synth.ffn_lognormal(rank)
    if workload in ("weight_tiles_fp8", "weight_rotated"):
        return synth.weight_outliers(seed=1 + 1000 * rank)
    gen, _, _ = synth.WORKLOADS[workload]
    base = {"tiny_weight": 0, "weight_outliers": 1, "activations_t3": 2, "weight_x50": 4}[workload]
    return gen(seed=base + 1000 * rank)


# ---------------------------------------------------------------------------
# byte accounting
# ---------------------------------------------------------------------------

def kernel_bytes(sizes, rows: int, cols: int):
    """Algorithmic bytes of (quantize, dequantize-to-bf16) for one scheme.
    sizes = (code, scale, zero point, tensor scale) bytes."""
    cb, sb, zb, tb = sizes
    x = 2 * rows * cols
    q = x + cb + sb + zb + tb
    dq = cb + sb + zb + tb + x
    return q, dq


def aggregate(bytes_per_step_per_rank: float, n_ranks: int, max_ms_per_step: float) -> float:
    """Whole-job GB/s: every rank moves the same bytes per step; the slowest rank sets the time."""
    return bytes_per_step_per_rank * n_ranks / (max_ms_per_step * 1e-3) / 1e9


def reduce_max(value: float, device=None) -> float:
    """Max of a float over ranks (identity without a process group)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if device is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.lines = []
        self.proc = None
        self.t_on = self.t_off = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "20",
                 "-i", str(self.gpu)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        self._t = threading.Thread(target=self._read, daemon=True)
        self._t.start()
        t0 = time.time()
        while not self.lines and time.time() - t0 < 5:
            time.sleep(0.01)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark_on(self):
        self.t_on = time.time()

    def mark_off(self):
        self.t_off = time.time()

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.05)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for t, line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            rows.append((t, parts))
        window = [p for t, p in rows if self.t_on - 0.025 <= t <= self.t_off + 0.025]
        use = window or [p for _, p in rows]

        def num(s):
            try:
                return float(s)
            except ValueError:
                return math.nan

        sm = [num(p[2]) for p in use]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for p in use:
            for name, v in zip(names, p[6:10]):
                if v.strip().lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(num(p[3]) for p in use) if use else None,
                "reasons": sorted(reasons),
                "samples": len(use), "samples_in_timed_region": len(window)}


# ---------------------------------------------------------------------------
# roofline inputs
# ---------------------------------------------------------------------------

def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def kernel_src_hash() -> str:
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "block_scaled_bit_bq_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(label: str, workload: str):
    """DRAM bytes per launch of a kernel from the committed ncu summary, if that summary
    was taken on the current kernel sources; else None."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.txt")
    if not os.path.exists(p):
        return None
    cur = kernel_src_hash()
    for line in open(p):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        kv = dict(item.split("=", 1) for item in line.split() if "=" in item)
        if kv.get("workload") == workload and kv.get("kernel") == label and kv.get("src_hash") == cur:
            return float(kv["dram_bytes_per_launch"])
    return None


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def run_ours(args, rank: int, world: int, local_rank: int):
    import block_scaled_bit_bq_b200 as bq
    from block_scaled_bit_bq_b200 import Scheme

    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    schemes = [(lab, Scheme(*a)) for lab, a in WORKLOADS[args.workload]]
    x_host = gen_input(args.workload, rank)
    rows, cols = x_host.shape
    signs = rotation_signs(args.workload, cols)
    sign_bits = None if signs is None else bq.pack_sign_bits(signs, device)
    per_scheme_bytes = [kernel_bytes(bq.bq_buffer_sizes(s, rows, cols), rows, cols) for _, s in schemes]
    if signs is not None:
        # the sign words are read by both kernels
        per_scheme_bytes = [(q + cols // 8, d + cols // 8) for q, d in per_scheme_bytes]
    step_bytes = sum(q + d for q, d in per_scheme_bytes)

    # buffer sets: inputs + outputs of every kernel, rotated so that each step touches
    # memory last used more than 4 x L2 ago
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    set_bytes = step_bytes
    n_sets = max(2, math.ceil(4 * l2 / set_bytes) + 1)
    n_sets = min(n_sets, max(2, int(0.5 * torch.cuda.mem_get_info(device)[0] // max(set_bytes, 1))))
    x_dev = x_host.to(device)
    sets = []
    for i in range(n_sets):
        xi = x_dev if i == 0 else x_dev.clone()
        outs = [bq.alloc_outputs(s, rows, cols, device, stats=True) for _, s in schemes]
        deqs = [torch.empty((rows, cols), dtype=torch.bfloat16, device=device) for _ in schemes]
        sets.append((xi, outs, deqs))
    stream = torch.cuda.current_stream(device)
    # the schemes of a step are independent: with two or more, they run as two lanes
    # (even schemes on the launching stream, odd ones on a side stream, each lane with its
    # own workspace), forked and joined inside the step, so one lane's kernels fill the
    # other's ramp and tail
    n_lanes = 1 if (args.serial or len(schemes) < 2) else 2
    wss = [bq.new_workspace(device) for _ in range(n_lanes)]
    side = torch.cuda.Stream(device) if n_lanes > 1 else None
    ws = wss[0]

    def launch(j, kind, i, st, ws=ws):
        """Kernel `kind` ("quantize" / "dequantize" / "qsnr") of scheme j on buffer set i."""
        xi, outs, deqs = sets[i % n_sets]
        s, q = schemes[j][1], outs[j]
        if sign_bits is not None and kind == "quantize":
            bq.bq_quantize_rt(xi, s, None, sign_bits, q.codes, q.scales, q.zero_points, q.stats, ws, st)
        elif sign_bits is not None and kind == "dequantize":
            bq.bq_dequantize_rt(q.codes, q.scales, q.zero_points, rows, cols, s, None, sign_bits, deqs[j], st)
        elif kind == "quantize":
            bq.bq_quantize(xi, s, q.codes, q.scales, q.zero_points, q.tensor_scale, q.stats, ws, st)
        elif kind == "dequantize":
            bq.bq_dequantize(q.codes, q.scales, q.zero_points, q.tensor_scale, rows, cols, s, deqs[j], st)
        else:
            bq.bq_qsnr(xi, q.codes, q.scales, q.zero_points, q.tensor_scale, s, q.stats, ws, st)

    def step(i, st=None):
        st = st or stream
        if n_lanes == 1:
            for j in range(len(schemes)):
                launch(j, "quantize", i, st)
                launch(j, "dequantize", i, st)
            return
        side.wait_stream(st)
        for j in range(len(schemes)):
            lane_st, lane_ws = (st, wss[0]) if j % 2 == 0 else (side, wss[1])
            launch(j, "quantize", i, lane_st, lane_ws)
            launch(j, "dequantize", i, lane_st, lane_ws)
        st.wait_stream(side)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(device)

    def capture(fn):
        """A CUDA graph of fn(stream) (captured on a side stream, replayed on `stream`)."""
        g = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream(device)
        cap.wait_stream(stream)
        with torch.cuda.graph(g, stream=cap):
            fn(cap)
        torch.cuda.synchronize(device)
        return g

    # The K timed steps are captured once into a CUDA graph and replayed once inside the
    # timed region, so host-side launch overhead does not enter the device time.
    graph = None
    if not args.eager:
        graph = capture(lambda st: [step(args.warmup + i, st) for i in range(args.steps)])
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    sampler = ClockSampler(vis.split(",")[local_rank].strip() if vis else device.index)
    if rank == 0:
        sampler.start()
    barrier(device)
    torch.cuda.synchronize(device)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    sampler.mark_on()
    t0.record(stream)
    if graph is not None:
        graph.replay()
    else:
        for i in range(args.steps):
            step(args.warmup + i)
    t1.record(stream)
    torch.cuda.synchronize(device)
    sampler.mark_off()
    barrier(device)
    clocks = sampler.stop() if rank == 0 else None
    ms = t0.elapsed_time(t1) / args.steps
    ms_max = reduce_max(ms, device)

    # QSNR of the last timed step (device sums read back before the per-kernel timing,
    # whose standalone QSNR launches rewrite them)
    qsnr = {}
    xi, outs, _ = sets[(args.warmup + args.steps - 1) % n_sets]
    for (lab, _), q in zip(schemes, outs):
        st = q.stats.cpu().tolist()
        qsnr[lab] = {"db": bq.bq_stats_qsnr_db(st), "mean_kappa": (st[2] / st[4]) if st[4] else None}

    # Per-kernel launch durations: each kernel of the step alone, K launches back to back
    # over the same rotating buffer sets (a graph of them, or eager), between two events
    # on the launching stream. (Events between the kernels of one graph would add their
    # own gaps to every interval.)
    n_k = 2 * len(schemes)
    n_per = max(8, min(args.steps, 64))
    kernels = []
    for j, (lab, s) in enumerate(schemes):
        qb, db = per_scheme_bytes[j]
        # the standalone QSNR pass (not part of the step) reads what quantize reads and writes
        kinds = (("quantize", qb), ("dequantize", db), ("qsnr", qb))
        if sign_bits is not None:
            kinds = kinds[:2]            # the rotated schemes have no standalone QSNR pass
        for kind, nbytes in kinds:
            def seq(st, j=j, kind=kind):
                for i in range(n_per):
                    launch(j, kind, args.warmup + i, st)
            seq(stream)                                  # warm
            g = None if args.eager else capture(seq)
            k0 = torch.cuda.Event(enable_timing=True)
            k1 = torch.cuda.Event(enable_timing=True)
            k0.record(stream)
            if g is not None:
                g.replay()
            else:
                seq(stream)
            k1.record(stream)
            torch.cuda.synchronize(device)
            kms = reduce_max(k0.elapsed_time(k1) / n_per, device)
            kernels.append({"kernel": f"{kind}:{lab}", "bytes": nbytes, "ms": kms,
                            "gbs": nbytes / (kms * 1e-3) / 1e9})
            del g
    dom = max((k for k in kernels if not k["kernel"].startswith("qsnr:")), key=lambda k: k["ms"])
    peak, peak_kind = measured_peaks()

    # end to end: pinned host input in, quantized outputs + sums out, every step. Steps
    # alternate between two device buffer sets, so the input copy of one step, the
    # kernels of the previous one and the output copy of the one before that overlap
    # (host-to-device and device-to-host copies on their own streams, ordered by events).
    e2e = None
    if not args.no_e2e:
        x_pin = x_host.pin_memory()
        n_buf = 2
        host_outs = []          # per buffer set: per scheme: (device tensor, pinned host tensor)
        d2h = 0
        for k in range(n_buf):
            per = []
            for q in sets[k][1]:
                hs = []
                for t in (q.codes, q.scales, q.zero_points, q.tensor_scale, q.stats):
                    if t is None:
                        continue
                    hs.append((t, torch.empty(t.shape, dtype=t.dtype).pin_memory()))
                    if k == 0:
                        d2h += t.numel() * t.element_size()
                per.append(hs)
            host_outs.append(per)
        h2d = x_pin.numel() * x_pin.element_size()
        s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
        ev_in = [torch.cuda.Event() for _ in range(n_buf)]
        ev_comp = [torch.cuda.Event() for _ in range(n_buf)]
        ev_out = [torch.cuda.Event() for _ in range(n_buf)]

        def e2e_step(i):
            k = i % n_buf
            s_in.wait_event(ev_comp[k])          # set k's input is no longer read
            with torch.cuda.stream(s_in):
                sets[k][0].copy_(x_pin, non_blocking=True)
            ev_in[k].record(s_in)
            stream.wait_event(ev_in[k])
            stream.wait_event(ev_out[k])         # set k's outputs are copied out
            step(k, stream)
            ev_comp[k].record(stream)
            s_out.wait_event(ev_comp[k])
            with torch.cuda.stream(s_out):
                for hs in host_outs[k]:
                    for t, h in hs:
                        h.copy_(t, non_blocking=True)
            ev_out[k].record(s_out)

        def e2e_run(n):
            s_in.wait_stream(stream)
            s_out.wait_stream(stream)
            for i in range(n):
                e2e_step(i)
            stream.wait_stream(s_out)

        e2e_run(max(2, args.warmup))
        torch.cuda.synchronize(device)
        barrier(device)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        n_e2e = max(2, min(args.steps, 50))
        e2e_run(n_e2e)
        e1.record(stream)
        torch.cuda.synchronize(device)
        e_ms = reduce_max(e0.elapsed_time(e1) / n_e2e, device)
        e2e = {"value": aggregate(step_bytes, world, e_ms), "unit": "GB/s", "ms_per_step": e_ms,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": n_e2e,
               "pipeline": "two buffer sets: a step's input copy, the previous step's kernels and the "
                           "output copy of the one before overlap (copies on their own streams)"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args.workload, schemes_args=WORKLOADS[args.workload], x_host=x_host,
                           budget_s=args.cpu_seconds, signs=signs)

    value = aggregate(step_bytes, world, ms_max)
    if rank != 0:
        return None
    traffic = ncu_traffic(dom["kernel"], args.workload)
    out = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_max,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic",
        "config": {
            "workload": f"{args.workload} {rows}x{cols} bf16: " + " + ".join(l for l, _ in schemes)
                        + ("; randomized full-row Hadamard rotation," if signs is not None else ";")
                        + " quantize with fused QSNR/kappa, then dequantize to bf16",
            "rows": rows, "cols": cols,
            "bytes_per_step_per_gpu": step_bytes,
            "l2": f"inputs larger than L2: {n_sets} rotating buffer sets of {set_bytes / 2**20:.1f} MiB",
            "parallelism": f"dp{world} (one independent tensor per GPU, no collective on the data path)",
            "launch": "eager" if graph is None else "CUDA graph of the K timed steps",
            "streams": (f"{n_lanes} (the step's independent schemes alternate between two streams, "
                        "forked and joined inside the step)") if n_lanes > 1 else "1",
            "kernel_timing": f"each kernel alone, {n_per} launches back to back over the rotating sets",
        },
        "pct_hbm_peak": round(100.0 * value / world / peak, 2),
        "roofline": {"bound": "hbm", "kernel": dom["kernel"], "achieved": round(dom["gbs"], 1),
                     "peak": peak, "unit": "GB/s", "frac": round(dom["gbs"] / peak, 4),
                     "traffic": traffic, "algorithmic_bytes": dom["bytes"], "peak_source": peak_kind},
        "kernels": [{k: (round(v, 4) if isinstance(v, float) else v) for k, v in kk.items()} for kk in kernels],
        "qsnr": qsnr,
        # quantize: one kernel, plus the range pass for per-tensor and NV scales; dequantize: one
        "gpu_launches": args.steps * sum((2 if s.gran in ("tensor", "nv") else 1) + 1 for _, s in schemes),
        "e2e": e2e,
        "cpu_baseline": cpu,
        "clocks": clocks,
    }
    return out


# ---------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline leg and the reference arm)
# ---------------------------------------------------------------------------

def oracle_step(xb: np.ndarray, schemes_args, signs=None):
    import oracle
    for _, a in schemes_args:
        s = oracle.Scheme(*a[:5])
        if signs is not None:
            r = oracle.quantize_rt(xb, s, signs=signs, stats=True)
            xh = oracle.dequantize_rt(r["codes"], r["scales"], r["zps"], xb.shape[0], xb.shape[1], s, signs=signs)
        else:
            r = oracle.quantize(xb, s, stats=True)
            xh = oracle.dequantize(r["codes"], r["scales"], r["zps"], r["tensor_scale"], xb.shape[0], xb.shape[1], s)
        oracle.to_bf16_array(xh)


def oracle_bytes(schemes_args, rows, cols):
    import oracle
    tot = 0
    for _, a in schemes_args:
        q, d = kernel_bytes(oracle.buffer_sizes(oracle.Scheme(*a[:5]), rows, cols), rows, cols)
        tot += q + d
    return tot


def cpu_baseline(workload, schemes_args, x_host, budget_s=10.0, rows_per_step=None, signs=None):
    """Time the oracle, as it stands, on this host (one thread) over whole steps of a
    row sample of the workload tensor, until budget_s is spent (at least 2 steps)."""
    xb = synth.bf16_bits(x_host)
    rows, cols = xb.shape
    if rows_per_step is None:
        t = time.perf_counter()
        oracle_step(xb[: max(1, rows // 32)], schemes_args, signs)
        per_row = (time.perf_counter() - t) / max(1, rows // 32)
        rows_per_step = int(min(rows, max(16, budget_s / 4 / max(per_row, 1e-9))))
    sample = xb[:rows_per_step]
    nbytes = oracle_bytes(schemes_args, rows_per_step, cols)
    t0 = time.perf_counter()
    n = 0
    while True:
        oracle_step(sample, schemes_args, signs)
        n += 1
        if n >= 2 and time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": round(nbytes * n / dt / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"first {rows_per_step} of {rows} rows of the {workload} tensor, {n} whole steps "
                      f"(quantize + dequantize of every scheme) in {dt:.1f} s, single thread"}


def run_reference(args, rank: int):
    if rank != 0:
        return None
    schemes_args = WORKLOADS[args.workload]
    x_host = gen_input(args.workload, 0)
    xb = synth.bf16_bits(x_host)
    rows, cols = xb.shape
    signs = rotation_signs(args.workload, cols)
    # rows per step so that warmup + steps take about args.cpu_seconds * 6 in total
    t = time.perf_counter()
    oracle_step(xb[: max(1, rows // 32)], schemes_args, signs)
    per_row = (time.perf_counter() - t) / max(1, rows // 32)
    total_budget = max(30.0, 6 * args.cpu_seconds)
    rows_per_step = int(min(rows, max(16, total_budget / (args.steps + args.warmup) / max(per_row, 1e-9))))
    sample = xb[:rows_per_step]
    nbytes = oracle_bytes(schemes_args, rows_per_step, cols)
    for _ in range(args.warmup):
        oracle_step(sample, schemes_args, signs)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(sample, schemes_args, signs)
    dt = time.perf_counter() - t0
    value = nbytes * args.steps / dt / 1e9
    desc = (f"first {rows_per_step} of {rows} rows of the {args.workload} tensor per step, "
            f"{args.steps} steps in {dt:.1f} s, single thread")
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 4),
        "unit": "GB/s",
        "n_gpus": 1,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": f"{args.workload} {rows}x{cols} bf16: " + " + ".join(l for l, _ in schemes_args)
                   + "; quantize with QSNR/kappa, then dequantize to bf16 (CPU oracle)",
                   "rows": rows, "cols": cols, "parallelism": "host, one thread"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": desc},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=list(WORKLOADS), default="weight_outliers")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--serial", action="store_true", help="run the step's schemes one after another on one stream")
    ap.add_argument("--eager", action="store_true", help="launch the timed steps one by one instead of as a CUDA graph")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        out = run_reference(args, rank)
        if out is not None:
            print(json.dumps(out), flush=True)
        return

    pg = False
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
        pg = True
    try:
        out = run_ours(args, rank, world, local_rank)
    finally:
        if pg:
            import torch.distributed as dist
            dist.destroy_process_group()
    if out is not None:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
