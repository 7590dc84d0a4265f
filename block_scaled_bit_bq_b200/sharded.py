"""One tensor split by rows across the ranks of a process group.

Every granularity but per-tensor is row-local, so each rank quantizes its own row block
with no communication. Per-tensor and NV schemes need the whole tensor's range before
the quantize pass: each rank takes its block's range (bq_tensor_range), one all-reduce
combines them (MAX of amax and of max, MIN of min: one MAX over [amax, -min, max]), and
each rank runs the quantize pass against the combined range (bq_quantize_with_range).
The QSNR and crest-factor sums combine with one more all-reduce (SUM of err2, x2, the
kappa sum and the unit count; MAX of the kappa maximum). A per-tensor scheme's single
kappa is formed from the combined sums: amax / sqrt(x2 / n).

The kernels do all the arithmetic; this module only orders the calls and the two
collectives ("INT vs FP at fine granularity" §2.1 for the per-tensor AbsMax scale, §4.1
for QSNR and kappa). Collectives run on the group's backend: NCCL over NVLink between
GPUs, gloo in the CPU tests of the combine steps.
"""

from __future__ import annotations

import math

import torch

from . import (Quantized, Scheme, alloc_outputs, bq_quantize, bq_quantize_with_range, bq_tensor_range,
               bq_workspace_size, new_workspace)

NEEDS_RANGE = ("tensor", "nv")


def _all_reduce(t: torch.Tensor, op, group) -> torch.Tensor:
    """all-reduce in place where the group's backend takes the tensor's device (gloo takes
    host tensors: a device tensor goes through a host copy)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return t
    if t.is_cuda and dist.get_backend(group) == "gloo":
        h = t.cpu()
        dist.all_reduce(h, op=op, group=group)
        t.copy_(h)
    else:
        dist.all_reduce(t, op=op, group=group)
    return t


def combine_ranges(local: torch.Tensor, group=None) -> torch.Tensor:
    """The whole tensor's {amax, min, max} from each rank's {amax, min, max} (fp32 [3],
    any device the group's backend serves): one all-reduce(MAX) of [amax, -min, max]."""
    import torch.distributed as dist
    t = torch.stack([local[0], -local[1], local[2]]).to(torch.float32)
    _all_reduce(t, dist.ReduceOp.MAX, group)
    return torch.stack([t[0], -t[1], t[2]])


def combine_stats(local: torch.Tensor, per_tensor_amax: float | None, n_elems_total: int,
                  group=None) -> torch.Tensor:
    """Whole-tensor stats (float64 [5]: err2, x2, kappa sum, kappa max, units) from each
    rank's stats of its block. per_tensor_amax: the combined amax of a per-tensor scheme
    (its one kappa is formed from the combined sums), else None."""
    import torch.distributed as dist
    s = local.to(torch.float64).clone()
    sums = torch.stack([s[0], s[1], s[2], s[4]])
    mx = s[3:4].clone()
    _all_reduce(sums, dist.ReduceOp.SUM, group)
    _all_reduce(mx, dist.ReduceOp.MAX, group)
    out = torch.stack([sums[0], sums[1], sums[2], mx[0], sums[3]])
    if per_tensor_amax is not None:
        x2 = float(out[1])
        k = per_tensor_amax / math.sqrt(x2 / n_elems_total) if x2 > 0.0 else 0.0
        out[2], out[3], out[4] = k, k, (1.0 if x2 > 0.0 else 0.0)
    return out


def quantize_rows_shard(x_shard: torch.Tensor, scheme: Scheme, total_rows: int, group=None, stats: bool = True,
                        workspace: torch.Tensor | None = None) -> tuple[Quantized, torch.Tensor | None]:
    """Quantize this rank's row block x_shard (bf16 [rows_here, cols] on its GPU) of a
    tensor of total_rows rows split across the group. Returns the block's outputs (codes,
    scales, zero points and the tensor scale, exactly the rows of a whole-tensor
    bq_quantize) and the whole tensor's stats (float64 [5] on the device, or None)."""
    s = scheme.resolved()
    rows, cols = x_shard.shape
    x_shard = x_shard.contiguous()
    q = alloc_outputs(s, rows, cols, x_shard.device, stats)
    if workspace is None and (stats or s.gran in NEEDS_RANGE):
        workspace = new_workspace(x_shard.device)
    amax = None
    if s.gran in NEEDS_RANGE:
        local = torch.zeros(3, dtype=torch.float32, device=x_shard.device)
        if rows > 0:
            bq_tensor_range(x_shard, s, local, workspace)
        rng = combine_ranges(local, group).contiguous()
        bq_quantize_with_range(x_shard, s, rng, q.codes, q.scales, q.zero_points, q.tensor_scale,
                               q.stats if stats else None, workspace if stats else None)
        amax = float(rng[0]) if s.gran == "tensor" else None
    else:
        bq_quantize(x_shard, s, q.codes, q.scales, q.zero_points, q.tensor_scale, q.stats if stats else None,
                    workspace if (stats or bq_workspace_size(s, rows, cols, stats) > 0) else None)
    tot = None
    if stats:
        tot = combine_stats(q.stats, amax, total_rows * cols, group)
    return q, tot
