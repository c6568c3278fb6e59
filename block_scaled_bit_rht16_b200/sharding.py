"""Row sharding of the quantizer across ranks (one process per GPU, torch.distributed).

Blocks are independent along rows, so a tensor split into contiguous row ranges quantizes
with no data exchange, except for two reductions:
  * the E4M3 two-level scale needs the amax of the whole rotated tensor ("低精度量化技术：IF4…",
    section 3.2). Each rank computes its alpha_r = RN(A_r / RN(qmax * 448)); rounding is
    monotonic, so max_r alpha_r is exactly the alpha of the whole tensor -- one all-reduce(MAX)
    of a single float, after which every rank quantizes with the tensor scale given;
  * statistics: the raw FP64 records add up (all-reduce(SUM) of 24 doubles).
Stochastic rounding stays identical to the unsharded tensor because its counter uses the
global element index (row offset r0 passed in).

The compute steps are passed in as callables so the same logic runs with the CUDA library on
GPUs and, in the tests, with the CPU oracle on gloo ranks.
"""
from dataclasses import dataclass
from typing import Callable

import torch
import torch.distributed as dist


def row_range(rows: int, rank: int, world: int, multiple: int = 1):
    """Contiguous [r0, r1) for `rank` of `world`; boundaries are multiples of `multiple`
    (16 for the dual orientation, whose column blocks span 16 rows)."""
    if rows % multiple:
        raise ValueError("rows must be a multiple of %d" % multiple)
    units = rows // multiple
    per, extra = divmod(units, world)
    u0 = rank * per + min(rank, extra)
    u1 = u0 + per + (1 if rank < extra else 0)
    return u0 * multiple, u1 * multiple


def global_tensor_scale(local_alpha: float, group=None) -> float:
    """max over ranks of the per-rank E4M3 tensor scale (= the whole tensor's scale)."""
    t = torch.tensor([float(local_alpha)], dtype=torch.float32)
    if dist.get_backend(group) == "nccl":
        t = t.cuda()
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


def global_stats_raw(local_raw, group=None):
    """Sum of the ranks' raw statistics records (FP64)."""
    t = torch.as_tensor(local_raw, dtype=torch.float64).clone()
    if dist.get_backend(group) == "nccl":
        t = t.cuda()
    dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
    return t.cpu().numpy()


@dataclass
class ShardSteps:
    """Compute steps for one rank's row range [r0, r1) of the tensor."""
    tensor_scale: Callable[[], float]                  # local alpha (E4M3 configurations)
    quantize: Callable[[object], object]               # quantize(alpha or None) -> result


def quantize_rows_sharded(steps: ShardSteps, e4m3_computed: bool, group=None):
    """One rank's part of a row-sharded quantization. With an E4M3 scale computed from the data,
    the ranks agree on the global tensor scale first; otherwise no communication happens."""
    alpha = None
    if e4m3_computed:
        alpha = global_tensor_scale(steps.tensor_scale(), group)
    return steps.quantize(alpha)
