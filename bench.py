"""Benchmark of the block-scaled quantization hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload ffn_lognormal|weight_outliers|tiny_weight|activations_t3|ffn_mx_family|
                                ffn_mx_gemm_operands|weight_tiles_fp8|weight_rotated|weight_x50]
                    [--tensors T]

The default workload is the FFN set at full size: 64 bf16 tensors of 4096 x 11008
(N(0, 1) times a per-row lognormal(0, 0.5) gain, seeds 3..66; the Llama-7B FFN shape of
"INT vs FP at fine granularity" §4.2) under MXINT8 and MXFP8 E4M3 (block 32 along rows,
UE8M0 scales).

A step is one pass of the quantize path over the workload's tensors: for every tensor
and every scheme, the quantize with the fused QSNR and crest-factor sums (bf16 load,
optional block-16 rotation, ranges, scales, codes, packing and the QSNR partial sums;
per-tensor and NV schemes take their range pass first). The FFN set takes one
bq_quantize_batch launch per scheme over its 64 tensors (--per-tensor: one bq_quantize
call per tensor); the other workloads one bq_quantize call per scheme.
value: quantize GB/s = algorithmic bytes of every quantize call of a step (x read once,
codes, scales, zero points and tensor scales written) / step time, summed over ranks
(weak scaling: each rank owns its own tensors), with inputs resident in HBM. The 64
distinct FFN tensors (5.8 GB) already exceed 4 x L2; single-tensor workloads rotate over
enough copies that every step reads data last touched more than 4 x L2 ago.
full_path: the same with the dequantize of every result to bf16 added to the step.
kernels: each kernel alone (quantize; for per-tensor / NV schemes also the range pass
and the quantize pass separately; dequantize; the standalone QSNR pass), launches back
to back over inputs rotating with a reuse distance of more than 4 x L2 of that
kernel's own bytes, as a CUDA graph replayed once untimed and once timed.
e2e: quantize GB/s when every step also copies its inputs from pinned host memory and
reads the codes, scales, zero points, tensor scales and QSNR sums back to the host.

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
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "quantize GB/s (bytes in+out) and % of B200 HBM peak; QSNR dB matching oracle"
# the sources the quantize kernels are built from (quant_flat.cu and what it includes): a traffic
# figure is used only while none of them has changed since its capture
KERNEL_SOURCES = ("common.cuh", "internal.h", "quant_flat.cu", "quant_ops.cuh", "rot.cuh", "rot64.cuh", "tma.cuh")

# workload -> list of (label, scheme args)
WORKLOADS = {
    "ffn_lognormal": [("mxint8", ("int8_sym", "mx", 32, "ue8m0", False)),
                      ("mxfp8_e4m3", ("e4m3", "mx", 32, "ue8m0", False))],
    "weight_outliers": [("uint4_g128_asym", ("uint4_asym", "group", 128, "fp16", False)),
                        ("int8_row_sym", ("int8_sym", "row", 0, "fp32", False))],
    "tiny_weight": [("int8_tensor_sym", ("int8_sym", "tensor", 0, "fp32", False)),
                    ("int4_g64_sym", ("int4_sym", "group", 64, "fp32", False))],
    "activations_t3": [("e4m3_tensor", ("e4m3", "tensor", 0, "fp32", False)),
                       ("e5m2_tensor", ("e5m2", "tensor", 0, "fp32", False)),
                       ("e4m3_token", ("e4m3", "row", 0, "fp32", False)),
                       ("e5m2_token", ("e5m2", "row", 0, "fp32", False))],
    # the rest of the MX family on the FFN tensors (MXFP4 and MXFP6)
    "ffn_mx_family": [("mxfp4", ("e2m1", "mx", 32, "ue8m0", False)),
                      ("mxfp6_e2m3", ("e2m3", "mx", 32, "ue8m0", False)),
                      ("mxfp6_e3m2", ("e3m2", "mx", 32, "ue8m0", False))],
    # the DeepSeek-V3 FP8 recipe on the 4096 x 4096 outlier weight: E4M3 with one fp32
    # scale per 128 x 128 tile (weights), and per 1 x 128 tile (the activation tiling)
    "weight_tiles_fp8": [("e4m3_tile128x128", ("e4m3", "tile2d", 128, "fp32", False)),
                         ("e4m3_tile1x128", ("e4m3", "group", 128, "fp32", False))],
    # GEMM operands: MXFP8 and MXFP4 of the FFN tensors with the block scales written in
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

# block-scaled GEMM workloads: D = A B^T of the 8192 x 8192 activations (Student-t(3) with
# outlier channels) and an 8192 x 8192 weight, both quantized (GEMM-layout scales)
GEMM_WORKLOADS = {"gemm_mxfp8": ("e4m3", "mx"), "gemm_nvfp4": ("e2m1", "nv")}

FFN_WORKLOADS = ("ffn_lognormal", "ffn_mx_family", "ffn_mx_gemm_operands")
# tensors per step: the FFN set is 64 tensors; the other workloads are one tensor
DEFAULT_TENSORS = {"ffn_lognormal": 64, "ffn_mx_family": 64, "ffn_mx_gemm_operands": 64}

# workloads whose schemes all run after the randomized full-row rotation: sign seed
ROTATED = {"weight_rotated": 21}


def rotation_signs(workload: str, cols: int):
    """The workload's per-column sign flags (uint8 0/1), or None."""
    return synth.random_signs(cols, ROTATED[workload]) if workload in ROTATED else None


def gen_inputs(workload: str, rank: int, n_tensors: int):
    """The rank's tensors (CPU bf16). FFN: tensors t = 64 * rank + i (seed 3 + t), drawn in
    parallel; else one tensor with the workload's seed shifted by 1000 * rank."""
    if workload in FFN_WORKLOADS:
        ids = [n_tensors * rank + i for i in range(n_tensors)]
        with ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
            return list(ex.map(synth.ffn_lognormal, ids))
    if workload in ("weight_tiles_fp8", "weight_rotated"):
        return [synth.weight_outliers(seed=1 + 1000 * rank)]
    gen, _, _ = synth.WORKLOADS[workload]
    base = {"tiny_weight": 0, "weight_outliers": 1, "activations_t3": 2, "weight_x50": 4}[workload]
    return [gen(seed=base + 1000 * rank)]


# ---------------------------------------------------------------------------
# byte accounting
# ---------------------------------------------------------------------------

def kernel_bytes(sizes, rows: int, cols: int):
    """Algorithmic bytes of one scheme's kernels on one tensor: quantize (x read once,
    outputs written), the range pass alone (x read), dequantize to bf16 (codes and
    scales read, bf16 written), standalone QSNR (x, codes and scales read).
    sizes = (code, scale, zero point, tensor scale) bytes."""
    cb, sb, zb, tb = sizes
    x = 2 * rows * cols
    out = cb + sb + zb + tb
    return {"quantize": x + out, "range": x, "quantize_pass": x + out, "dequantize": out + x, "qsnr": x + out}


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

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.lines = []
        self.proc = None
        self.windows = []

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

    def mark(self, t_on: float, t_off: float):
        self.windows.append((t_on, t_off))

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
        window = [p for t, p in rows if any(a - 0.025 <= t <= b + 0.025 for a, b in self.windows)]
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
    """DRAM bytes (read + write) per launch of a kernel from the committed ncu summary, if
    that summary was taken on the current kernel sources; else None."""
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

def measured_tensor_peak(fmt: str):
    """Dense tensor-core peak for the GEMM's element type: the measured bf16 burst figure
    times the nominal ratio (FP8 2x, FP4 4x bf16)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    ratio = 4.0 if fmt == "e2m1" else 2.0
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f)["bf16_tflops"]) * ratio, "measured bf16 x nominal ratio"
    return 1590.0 * ratio, "fallback bf16 x nominal ratio"


def run_gemm_bench(args, rank: int, world: int, device):
    """TFLOP/s of bq_gemm (and of the library's block-scaled GEMM on the same operands)."""
    import block_scaled_bit_bq_b200 as bq
    from block_scaled_bit_bq_b200 import Scheme
    fmt, gran = GEMM_WORKLOADS[args.workload]
    s = Scheme(fmt, gran, layout="gemm")
    M = N = K = 8192
    a = synth.activations_t3(M, K, seed=2 + 1000 * rank)
    b = synth.weight_outliers(N, K, seed=41 + 1000 * rank)
    qa = bq.quantize(a.to(device), s, stats=False)
    qb = bq.quantize(b.to(device), s, stats=False)
    d = torch.empty((M, N), dtype=torch.bfloat16, device=device)
    stream = torch.cuda.current_stream(device)
    flops = 2.0 * M * N * K

    def time_fn(fn, reps):
        for _ in range(3):
            fn()
        barrier(device)
        torch.cuda.synchronize(device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(device)
        return reduce_max(e0.elapsed_time(e1) / reps, device)

    reps = max(5, args.steps)
    ms = time_fn(lambda: bq.bq_gemm(qa, qb, d), reps)
    lib = None
    F = torch.nn.functional
    if fmt == "e4m3" and hasattr(F, "scaled_mm") and hasattr(torch, "float8_e8m0fnu"):
        dt = torch.float8_e4m3fn

        def lib_gemm():
            return F.scaled_mm(qa.codes.view(dt), qb.codes.view(dt).t(),
                               qa.scales.view(torch.float8_e8m0fnu), F.ScalingType.BlockWise1x32,
                               qb.scales.view(torch.float8_e8m0fnu), F.ScalingType.BlockWise1x32,
                               swizzle_a=F.SwizzleType.SWIZZLE_32_4_4, swizzle_b=F.SwizzleType.SWIZZLE_32_4_4,
                               output_dtype=torch.bfloat16)
        try:
            lib_ms = time_fn(lib_gemm, reps)
            lib = {"kernel": "cuBLASLt scaled_mm (torch)", "ms": lib_ms, "tflops": flops / (lib_ms * 1e-3) / 1e12}
        except RuntimeError as e:
            lib = {"kernel": "cuBLASLt scaled_mm (torch)", "unavailable": str(e).splitlines()[0][:200]}
    elif fmt == "e2m1" and hasattr(F, "scaled_mm") and hasattr(torch, "float4_e2m1fn_x2") \
            and hasattr(F.ScalingType, "BlockWise1x16"):
        fp4, e4 = torch.float4_e2m1fn_x2, torch.float8_e4m3fn
        ca, cb = qa.codes.view(fp4), qb.codes.view(fp4).t()
        sa, sb = qa.scales.view(e4), qb.scales.view(e4)

        def lib_gemm():
            # the two-level NVFP4 form: block scales and each operand's tensor scale
            return F.scaled_mm(ca, cb, [sa, qa.tensor_scale], [F.ScalingType.BlockWise1x16, F.ScalingType.TensorWise],
                               [sb, qb.tensor_scale], [F.ScalingType.BlockWise1x16, F.ScalingType.TensorWise],
                               swizzle_a=[F.SwizzleType.SWIZZLE_32_4_4, F.SwizzleType.NO_SWIZZLE],
                               swizzle_b=[F.SwizzleType.SWIZZLE_32_4_4, F.SwizzleType.NO_SWIZZLE],
                               output_dtype=torch.bfloat16)
        def lib_gemm_blocks():
            # block scales only (the tensor scales would multiply the result)
            return F.scaled_mm(ca, cb, sa, F.ScalingType.BlockWise1x16, sb, F.ScalingType.BlockWise1x16,
                               swizzle_a=F.SwizzleType.SWIZZLE_32_4_4, swizzle_b=F.SwizzleType.SWIZZLE_32_4_4,
                               output_dtype=torch.bfloat16)
        for name, fn in (("cuBLASLt scaled_mm NVFP4 (torch)", lib_gemm),
                         ("cuBLASLt scaled_mm NVFP4, block scales only (torch)", lib_gemm_blocks)):
            try:
                lib_ms = time_fn(fn, reps)
                lib = {"kernel": name, "ms": lib_ms, "tflops": flops / (lib_ms * 1e-3) / 1e12}
                break
            except (RuntimeError, TypeError, ValueError) as e:
                lib = {"kernel": name, "unavailable": str(e).splitlines()[0][:200]}
    if rank != 0:
        return None
    peak, src = measured_tensor_peak(fmt)
    tf = flops / (ms * 1e-3) / 1e12
    return {
        "metric": "block-scaled GEMM TFLOP/s (bq_gemm, D = A B^T)", "value": round(tf * world, 2), "unit": "TFLOP/s",
        "n_gpus": world, "steps": reps, "warmup": 3, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": fmt, "data": "synthetic",
        "config": {"workload": f"{args.workload}: {M}x{N}x{K}, {fmt} {gran} block scales in the GEMM layout, bf16 out",
                   "operands": "A: activations_t3 8192x8192 (Student-t(3) with outlier channels); B: weight_outliers 8192x8192"},
        "roofline": {"bound": "tensor", "achieved": round(tf, 1), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(tf / peak, 4), "traffic": None, "peak_source": src},
        "library_gemm": lib, "gpu_launches": reps,
    }


def run_ours(args, rank: int, world: int, local_rank: int):
    import block_scaled_bit_bq_b200 as bq
    from block_scaled_bit_bq_b200 import Scheme

    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    if args.workload in GEMM_WORKLOADS:
        return run_gemm_bench(args, rank, world, device)
    schemes = [(lab, Scheme(*a)) for lab, a in WORKLOADS[args.workload]]
    n_tensors = args.tensors or DEFAULT_TENSORS.get(args.workload, 1)
    hosts = gen_inputs(args.workload, rank, n_tensors)
    rows, cols = hosts[0].shape
    signs = rotation_signs(args.workload, cols)
    sign_bits = None if signs is None else bq.pack_sign_bits(signs, device)
    kb = [kernel_bytes(bq.bq_buffer_sizes(s, rows, cols), rows, cols) for _, s in schemes]
    if signs is not None:
        # the sign words are read by both kernels
        kb = [{k: v + cols // 8 for k, v in d.items()} for d in kb]
    # per-tensor and NV schemes: the range pass and the quantize pass are two kernels
    two_pass = [s.resolved().gran in ("tensor", "nv") for _, s in schemes]

    # units: the device copies of the inputs that the steps and the kernel timing rotate
    # over. FFN: the distinct tensors. One-tensor workloads: enough copies that the
    # smallest kernel's reuse distance exceeds 4 x L2.
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    smallest = min(min(v for k, v in d.items() if k != "range") for d in kb)
    if len(hosts) > 1:
        srcs = hosts
    else:
        n_copies = max(2, math.ceil(4 * l2 / smallest) + 1)
        free = torch.cuda.mem_get_info(device)[0]
        unit_bytes = 2 * rows * cols * 2 + sum(d["quantize"] for d in kb)
        n_copies = min(n_copies, max(2, int(0.5 * free // unit_bytes)))
        srcs = hosts * n_copies
    n_units = len(srcs)
    # the units as one contiguous [n_units, rows, cols] tensor (a batch call takes it whole)
    X = torch.empty((n_units, rows, cols), dtype=torch.bfloat16, device=device)
    for u, h in enumerate(srcs):
        X[u].copy_(h)
    xs = [X[u] for u in range(n_units)]
    # FFN sets quantize all their tensors in one bq_quantize_batch launch per scheme
    batched = len(hosts) > 1 and not args.per_tensor and signs is None and not any(two_pass)
    if batched:
        qbs = [bq.alloc_batch_outputs(s, n_units, rows, cols, device, stats=True) for _, s in schemes]
        outs = [[qbs[j].tensor(u) for j in range(len(schemes))] for u in range(n_units)]
    else:
        qbs = None
        outs = [[bq.alloc_outputs(s, rows, cols, device, stats=True) for _, s in schemes] for _ in range(n_units)]
    deqs = [torch.empty((rows, cols), dtype=torch.bfloat16, device=device) for _ in range(n_units)]
    rngs = [torch.zeros(3, dtype=torch.float32, device=device) for _ in range(n_units)]
    stream = torch.cuda.current_stream(device)
    # the schemes of a step are independent: with two or more, they run as two lanes
    # (even schemes on the launching stream, odd ones on a side stream, each lane with its
    # own workspace), forked and joined inside the step, so one lane's kernels fill the
    # other's ramp and tail
    n_lanes = 1 if (args.serial or len(schemes) < 2) else 2
    wss = [bq.new_workspace(device) for _ in range(n_lanes)]
    side = torch.cuda.Stream(device) if n_lanes > 1 else None

    def launch(j, kind, u, st, ws):
        """Kernel `kind` of scheme j on unit u (mod n_units); "quantize_batch": every unit."""
        u %= n_units
        xi, q, s = xs[u], outs[u][j], schemes[j][1]
        if kind == "quantize_batch":
            qb = qbs[j]
            bq.bq_quantize_batch(X, s, qb.codes, qb.scales, qb.zero_points, qb.stats, ws, st)
        elif sign_bits is not None and kind == "quantize":
            bq.bq_quantize_rt(xi, s, None, sign_bits, q.codes, q.scales, q.zero_points, q.stats, ws, st)
        elif sign_bits is not None and kind == "dequantize":
            bq.bq_dequantize_rt(q.codes, q.scales, q.zero_points, rows, cols, s, None, sign_bits, deqs[u], st)
        elif kind == "quantize":
            bq.bq_quantize(xi, s, q.codes, q.scales, q.zero_points, q.tensor_scale, q.stats, ws, st)
        elif kind == "range":
            bq.bq_tensor_range(xi, s, rngs[u], ws, st)
        elif kind == "quantize_pass":
            bq.bq_quantize_with_range(xi, s, rngs[u], q.codes, q.scales, q.zero_points, q.tensor_scale, q.stats,
                                      ws, st)
        elif kind == "dequantize":
            bq.bq_dequantize(q.codes, q.scales, q.zero_points, q.tensor_scale, rows, cols, s, deqs[u], st)
        else:
            bq.bq_qsnr(xi, q.codes, q.scales, q.zero_points, q.tensor_scale, s, q.stats, ws, st)

    # units of step i: every FFN tensor, or the i-th copy of the one tensor
    def step_units(i):
        return list(range(n_units)) if len(hosts) > 1 else [i % n_units]

    def step(i, st=None, dequant=False):
        st = st or stream
        lanes = [(st, wss[0])] if n_lanes == 1 else [(st, wss[0]), (side, wss[1])]
        if n_lanes > 1:
            side.wait_stream(st)
        if batched:
            for j in range(len(schemes)):
                lane_st, lane_ws = lanes[j % n_lanes]
                launch(j, "quantize_batch", 0, lane_st, lane_ws)
                if dequant:
                    for u in step_units(i):
                        launch(j, "dequantize", u, lane_st, lane_ws)
        else:
            for u in step_units(i):
                for j in range(len(schemes)):
                    lane_st, lane_ws = lanes[j % n_lanes]
                    launch(j, "quantize", u, lane_st, lane_ws)
                    if dequant:
                        launch(j, "dequantize", u, lane_st, lane_ws)
        if n_lanes > 1:
            st.wait_stream(side)

    units_per_step = len(step_units(0))
    q_bytes = units_per_step * sum(d["quantize"] for d in kb)
    full_bytes = units_per_step * sum(d["quantize"] + d["dequantize"] for d in kb)

    for i in range(args.warmup):
        step(i, dequant=True)
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

    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    sampler = ClockSampler(vis.split(",")[local_rank].strip() if vis else device.index)
    if rank == 0:
        sampler.start()

    def timed(fn_graph, fn_eager, n):
        """Device ms per iteration of a graph replay (or eager loop) between two events."""
        barrier(device)
        torch.cuda.synchronize(device)
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        a = time.time()
        t0.record(stream)
        if fn_graph is not None:
            fn_graph.replay()
        else:
            fn_eager()
        t1.record(stream)
        torch.cuda.synchronize(device)
        sampler.mark(a, time.time())
        barrier(device)
        return reduce_max(t0.elapsed_time(t1) / n, device)

    # The K timed steps are captured once into a CUDA graph and replayed once inside the
    # timed region, so host-side launch overhead does not enter the device time.
    graph = None if args.eager else capture(lambda st: [step(args.warmup + i, st) for i in range(args.steps)])
    ms_max = timed(graph, lambda: [step(args.warmup + i) for i in range(args.steps)], args.steps)
    del graph

    # QSNR of the last timed step (read back before later launches rewrite the sums)
    qsnr = {}
    last = step_units(args.warmup + args.steps - 1)
    for j, (lab, _) in enumerate(schemes):
        dbs, kap = [], []
        for u in last:
            st = outs[u][j].stats.cpu().tolist()
            dbs.append(bq.bq_stats_to_db(st))
            if st[4]:
                kap.append(st[2] / st[4])
        qsnr[lab] = {"mean_db": statistics.fmean(dbs), "min_db": min(dbs), "max_db": max(dbs),
                     "mean_kappa": statistics.fmean(kap) if kap else None, "tensors": len(dbs)}

    # the whole path: quantize and dequantize of every tensor under every scheme
    n_full = max(2, min(args.steps, 10))
    g_full = None if args.eager else capture(
        lambda st: [step(args.warmup + i, st, dequant=True) for i in range(n_full)])
    ms_full = timed(g_full, lambda: [step(args.warmup + i, dequant=True) for i in range(n_full)], n_full)
    del g_full

    # Per-kernel launch durations: each kernel alone, n_per launches back to back over
    # the rotating units, between two events on the launching stream. (Events between
    # the kernels of one graph would add their own gaps to every interval.)
    n_per = max(8, min(64, 2 * n_units))
    kernels = []
    for j, (lab, s) in enumerate(schemes):
        kinds = ["quantize_batch", "quantize"] if batched else ["quantize"]
        if two_pass[j]:
            kinds += ["range", "quantize_pass"]
        kinds += ["dequantize"]
        if sign_bits is None:
            kinds += ["qsnr"]          # (the rotated schemes have no standalone QSNR pass)
        for kind in kinds:
            if kind == "quantize_pass":
                for u in range(n_units):       # every unit's range, for its quantize pass
                    launch(j, "range", u, stream, wss[0])

            reps = max(3, min(8, n_per)) if kind == "quantize_batch" else n_per

            def seq(st, j=j, kind=kind, reps=reps):
                for i in range(reps):
                    launch(j, kind, i, st, wss[0])
            seq(stream)                                  # warm
            g = None if args.eager else capture(seq)
            if g is not None:
                # the graph's first launch carries a one-time cost (~20 us, ~2 us a kernel
                # over these short sequences); a first replay keeps it out of the timing
                g.replay()
            kms = timed(g, lambda: seq(stream), reps)
            nbytes = kb[j]["quantize"] * n_units if kind == "quantize_batch" else kb[j][kind]
            reuse = nbytes if kind == "quantize_batch" else min(n_per, n_units) * kb[j][kind]
            kernels.append({"kernel": f"{kind}:{lab}", "bytes": nbytes, "ms": kms,
                            "gbs": nbytes / (kms * 1e-3) / 1e9, "reuse_distance_bytes": reuse,
                            **({"tensors": n_units} if kind == "quantize_batch" else {})})
            del g
    # the dominant kernel of the step: the slowest single kernel that the quantize step
    # launches (for two-pass schemes the range pass and the quantize pass count apart)
    is_two_pass = {lab: tp for (lab, _), tp in zip(schemes, two_pass)}

    def in_step(k):
        kind, lab = k["kernel"].split(":", 1)
        if batched:
            return kind == "quantize_batch"
        return kind in ("range", "quantize_pass") if is_two_pass[lab] else kind == "quantize"
    step_kernels = [k for k in kernels if in_step(k)]
    dom = max(step_kernels, key=lambda k: k["ms"])
    peak, peak_kind = measured_peaks()

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, bq, schemes, hosts, rows, cols, device, stream, wss, sign_bits, q_bytes, world)

    clocks = sampler.stop() if rank == 0 else None
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args.workload, WORKLOADS[args.workload], hosts[0], budget_s=args.cpu_seconds,
                           signs=signs)

    value = aggregate(q_bytes, world, ms_max)
    if rank != 0:
        return None
    traffic = ncu_traffic(dom["kernel"], args.workload)
    n_launch_q = sum(2 if tp else 1 for tp in two_pass)
    launches_per_step = len(schemes) if batched else units_per_step * n_launch_q
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
            "workload": (f"{args.workload}: {units_per_step} x bf16 {rows}x{cols} per step: "
                         + " + ".join(l for l, _ in schemes)
                         + ("; randomized full-row Hadamard rotation" if signs is not None else "")
                         + "; quantize with fused QSNR/kappa"),
            "tensors_per_step": units_per_step, "rows": rows, "cols": cols,
            "bytes_per_step_per_gpu": q_bytes,
            "l2": (f"inputs larger than L2: {n_units} distinct {'tensors' if len(hosts) > 1 else 'copies'} of "
                   f"{2 * rows * cols / 2**20:.1f} MiB rotate (L2 {l2 / 2**20:.0f} MiB)"),
            "parallelism": f"dp{world} (each GPU owns its own tensors, no collective on the data path)",
            "launch": ("eager" if args.eager else "CUDA graph of the K timed steps")
                      + ("; one bq_quantize_batch launch per scheme over the step's tensors" if batched
                         else "; one bq_quantize call per tensor and scheme"),
            "streams": (f"{n_lanes} (the step's independent schemes alternate between two streams, "
                        "forked and joined inside the step)") if n_lanes > 1 else "1",
            "kernel_timing": (f"each kernel alone, {n_per} launches back to back over the rotating inputs "
                              "(reuse distance per kernel in kernels[].reuse_distance_bytes)"),
        },
        "pct_hbm_peak": round(100.0 * value / world / peak, 2),
        "full_path": {"value": round(aggregate(full_bytes, world, ms_full), 2), "unit": "GB/s",
                      "ms_per_step": ms_full, "bytes_per_step_per_gpu": full_bytes,
                      "what": "quantize with fused QSNR/kappa, then dequantize to bf16, of every tensor and scheme"},
        "roofline": {"bound": "hbm", "kernel": dom["kernel"], "achieved": round(dom["gbs"], 1),
                     "peak": peak, "unit": "GB/s", "frac": round(dom["gbs"] / peak, 4),
                     "traffic": traffic, "algorithmic_bytes": dom["bytes"], "peak_source": peak_kind},
        "kernels": [{k: (round(v, 4) if isinstance(v, float) else v) for k, v in kk.items()} for kk in kernels],
        "qsnr": qsnr,
        "gpu_launches": args.steps * launches_per_step,
        "e2e": e2e,
        "cpu_baseline": cpu,
        "clocks": clocks,
    }
    return out


def run_e2e(args, bq, schemes, hosts, rows, cols, device, stream, wss, sign_bits, q_bytes, world):
    """Quantize GB/s end to end: each tensor's input is copied from pinned host memory and
    its codes, scales, zero points, tensor scale and QSNR sums are read back, every step.
    A ring of three device slots lets one tensor's input copy, another's kernels and a
    third's output copy run at the same time (copies on their own streams, ordered by
    events)."""
    n_slots = 3
    pins = [h.pin_memory() for h in hosts]
    slot_x = [torch.empty((rows, cols), dtype=torch.bfloat16, device=device) for _ in range(n_slots)]
    slot_q = [[bq.alloc_outputs(s, rows, cols, device, stats=True) for _, s in schemes] for _ in range(n_slots)]

    def out_tensors(qs):
        return [t for q in qs for t in (q.codes, q.scales, q.zero_points, q.tensor_scale, q.stats) if t is not None]

    host_out = [[torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in out_tensors(slot_q[k])]
                for k in range(n_slots)]
    h2d = sum(p.numel() * p.element_size() for p in pins[:1])
    d2h = sum(t.numel() * t.element_size() for t in out_tensors(slot_q[0]))
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev_in = [torch.cuda.Event() for _ in range(n_slots)]
    ev_comp = [torch.cuda.Event() for _ in range(n_slots)]
    ev_out = [torch.cuda.Event() for _ in range(n_slots)]
    for e in ev_comp + ev_out:
        e.record(stream)
    k_ring = [0]

    def one(u):
        k = k_ring[0] % n_slots
        k_ring[0] += 1
        s_in.wait_event(ev_comp[k])           # slot k's input is no longer read
        with torch.cuda.stream(s_in):
            slot_x[k].copy_(pins[u], non_blocking=True)
        ev_in[k].record(s_in)
        stream.wait_event(ev_in[k])
        stream.wait_event(ev_out[k])          # slot k's outputs are copied out
        for j, (_, s) in enumerate(schemes):
            q = slot_q[k][j]
            if sign_bits is not None:
                bq.bq_quantize_rt(slot_x[k], s, None, sign_bits, q.codes, q.scales, q.zero_points, q.stats,
                                  wss[0], stream)
            else:
                bq.bq_quantize(slot_x[k], s, q.codes, q.scales, q.zero_points, q.tensor_scale, q.stats, wss[0],
                               stream)
        ev_comp[k].record(stream)
        s_out.wait_event(ev_comp[k])
        with torch.cuda.stream(s_out):
            for t, h in zip(out_tensors(slot_q[k]), host_out[k]):
                h.copy_(t, non_blocking=True)
        ev_out[k].record(s_out)

    def run(n_steps):
        s_in.wait_stream(stream)
        s_out.wait_stream(stream)
        for _ in range(n_steps):
            for u in range(len(hosts)):
                one(u)
        stream.wait_stream(s_out)

    n_e2e = max(2, min(args.steps, 3 if len(hosts) > 1 else 50))
    run(1)
    torch.cuda.synchronize(device)
    barrier(device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    run(n_e2e)
    e1.record(stream)
    torch.cuda.synchronize(device)
    e_ms = reduce_max(e0.elapsed_time(e1) / n_e2e, device)
    return {"value": round(aggregate(q_bytes, world, e_ms), 2), "unit": "GB/s", "ms_per_step": e_ms,
            "h2d_bytes_per_step": h2d * len(hosts), "d2h_bytes_per_step": d2h * len(hosts), "steps": n_e2e,
            "pipeline": "three device slots: one tensor's input copy, another's quantize and a third's output "
                        "copy overlap (copies on their own streams)"}


# ---------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline leg and the reference arm)
# ---------------------------------------------------------------------------

def _blocks(rows: int, n: int):
    edges = [rows * i // n for i in range(n + 1)]
    return [(a, b) for a, b in zip(edges[:-1], edges[1:]) if b > a]


def oracle_step(xb: np.ndarray, schemes_args, signs=None, threads: int = 1):
    """Quantize (with QSNR / kappa sums) and dequantize to bf16 of one tensor under every
    scheme with the oracle. threads > 1 splits the rows into blocks run concurrently (the
    oracle's C calls release the interpreter lock); per-tensor and NV schemes first take
    the whole tensor's range (blocks' ranges combined), then quantize each block against it."""
    import oracle
    rows, cols = xb.shape
    blocks = _blocks(rows, threads)

    def one_block(args):
        (a, b), s, tr = args
        xp = xb[a:b]
        if signs is not None:
            r = oracle.quantize_rt(xp, s, signs=signs, stats=True)
            xh = oracle.dequantize_rt(r["codes"], r["scales"], r["zps"], b - a, cols, s, signs=signs)
        else:
            r = oracle.quantize(xp, s, tensor_range=tr, stats=True)
            xh = oracle.dequantize(r["codes"], r["scales"], r["zps"], r["tensor_scale"], b - a, cols, s)
        oracle.to_bf16_array(xh)

    with ThreadPoolExecutor(max_workers=max(1, threads)) as ex:
        for _, a in schemes_args:
            s = oracle.Scheme(*a[:5])
            tr = None
            if s.gran in ("tensor", "nv") and signs is None and len(blocks) > 1:
                parts = list(ex.map(lambda ab: oracle.tensor_range(xb[ab[0]:ab[1]], s.hadamard), blocks))
                tr = (max(p[0] for p in parts), min(p[1] for p in parts), max(p[2] for p in parts))
            list(ex.map(one_block, [(ab, s, tr) for ab in blocks]))


def oracle_bytes(schemes_args, rows, cols):
    """Algorithmic bytes of one oracle step: quantize and dequantize of every scheme."""
    import oracle
    tot = 0
    for _, a in schemes_args:
        d = kernel_bytes(oracle.buffer_sizes(oracle.Scheme(*a[:5]), rows, cols), rows, cols)
        tot += d["quantize"] + d["dequantize"]
    return tot


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def time_oracle(xb, schemes_args, budget_s, signs, threads):
    """Whole oracle steps on a row sample sized so the timing takes about budget_s."""
    rows, cols = xb.shape
    probe = max(threads, rows // 64)
    t = time.perf_counter()
    oracle_step(xb[:probe], schemes_args, signs, threads)
    per_row = (time.perf_counter() - t) / probe
    rows_per_step = int(min(rows, max(16 * threads, budget_s / 4 / max(per_row, 1e-9))))
    sample = xb[:rows_per_step]
    nbytes = oracle_bytes(schemes_args, rows_per_step, cols)
    t0 = time.perf_counter()
    n = 0
    while True:
        oracle_step(sample, schemes_args, signs, threads)
        n += 1
        if n >= 2 and time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return nbytes * n / dt / 1e9, rows_per_step, n, dt


def cpu_baseline(workload, schemes_args, x_host, budget_s=10.0, signs=None):
    """Time the oracle, as it stands, on this host: all cores (row blocks in parallel) and
    one thread, each over whole steps (quantize with QSNR / kappa sums, then dequantize, of
    every scheme) of a row sample of the workload's first tensor."""
    xb = synth.bf16_bits(x_host)
    rows, cols = xb.shape
    cores = host_cores()
    v_all, r_all, n_all, dt_all = time_oracle(xb, schemes_args, budget_s, signs, cores)
    v_one, r_one, n_one, dt_one = time_oracle(xb, schemes_args, budget_s, signs, 1)
    return {"value": round(v_all, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": (f"first {r_all} of {rows} rows of the {workload} tensor, {n_all} whole steps (quantize "
                       f"with QSNR/kappa + dequantize of every scheme) in {dt_all:.1f} s, rows split over "
                       f"{cores} threads"),
            "single_thread": {"value": round(v_one, 4), "unit": "GB/s", "cores": 1,
                              "sample": f"first {r_one} rows, {n_one} whole steps in {dt_one:.1f} s"}}


def run_reference(args, rank: int):
    if rank != 0:
        return None
    if args.workload in GEMM_WORKLOADS:
        return {"impl": "reference", "unavailable": "the GEMM workloads have no CPU arm (the oracle's float64 GEMM "
                                                   "reference serves the parity tests only)"}
    schemes_args = WORKLOADS[args.workload]
    x_host = gen_inputs(args.workload, 0, 1)[0]
    xb = synth.bf16_bits(x_host)
    rows, cols = xb.shape
    signs = rotation_signs(args.workload, cols)
    cores = host_cores()
    # rows per step so that warmup + steps take about args.cpu_seconds * 6 in total
    probe = max(cores, rows // 64)
    t = time.perf_counter()
    oracle_step(xb[:probe], schemes_args, signs, cores)
    per_row = (time.perf_counter() - t) / probe
    total_budget = max(30.0, 6 * args.cpu_seconds)
    rows_per_step = int(min(rows, max(16 * cores, total_budget / (args.steps + args.warmup) / max(per_row, 1e-9))))
    sample = xb[:rows_per_step]
    nbytes = oracle_bytes(schemes_args, rows_per_step, cols)
    for _ in range(args.warmup):
        oracle_step(sample, schemes_args, signs, cores)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(sample, schemes_args, signs, cores)
    dt = time.perf_counter() - t0
    value = nbytes * args.steps / dt / 1e9
    desc = (f"first {rows_per_step} of {rows} rows of the {args.workload} tensor per step, "
            f"{args.steps} steps in {dt:.1f} s, rows split over {cores} threads")
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
        "config": {"workload": f"{args.workload}: bf16 {rows}x{cols}: " + " + ".join(l for l, _ in schemes_args)
                   + "; quantize with QSNR/kappa, then dequantize to bf16 (CPU oracle)",
                   "rows": rows, "cols": cols, "parallelism": f"host, {cores} threads"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": desc},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=list(WORKLOADS) + list(GEMM_WORKLOADS), default="ffn_lognormal")
    ap.add_argument("--tensors", type=int, default=0, help="tensors per step (FFN workloads; default 64)")
    ap.add_argument("--per-tensor", action="store_true",
                    help="FFN sets: one bq_quantize call per tensor instead of one batch call per scheme")
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
