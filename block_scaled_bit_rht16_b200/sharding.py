"""Row sharding of the quantizer across ranks (one process per GPU, torch.distributed).

Blocks are independent along rows, so a tensor split into contiguous row ranges quantizes
with no data exchange, except for two reductions:
  * the E4M3 two-level scale needs the amax of the whole rotated tensor ("低精度量化技术：IF4…",
    section 3.2). Each rank computes its alpha_r = RN(A_r / RN(qmax * 448)); rounding is
    monotonic, so max_r alpha_r is exactly the alpha of the whole tensor -- one all-reduce(MAX)
    of a single float, after which every rank quantizes with the tensor scale given;
  * statistics: the raw FP64 records add up (all-reduce(SUM) of 24 doubles).
Stochastic rounding stays identical to the unsharded tensor: a shard quantizes its rows as a
tensor of their own (element indices from 0) with the seed from shard_sr_seed, which starts
the counter stream where those rows start in the whole tensor. This holds for the row
orientation. The column orientation of the dual dY pass indexes element (m, n) as n * M + m,
which depends on the whole tensor's M; a row-sharded dual pass with stochastic rounding on the
column orientation therefore draws differently from the unsharded one.

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


GAMMA = 0x9E3779B97F4A7C15   # SplitMix64's state increment (Steele, Lea & Flood 2014)


def shard_sr_seed(sr_seed: int, r0: int, cols: int) -> int:
    """The stochastic-rounding seed for rows [r0, ...) of a [rows, cols] tensor quantized on
    their own, such that every element draws what it draws inside the whole tensor.

    Element idx (row-major) takes 16-bit lane idx & 3 of output idx >> 2 of the SplitMix64
    stream whose state starts at the seed (with the stream number in bit 63) and advances by
    GAMMA per output. Row r0 starts at output r0 * cols / 4 (cols is a multiple of 4), so the
    shard's stream must start r0 * cols / 4 increments later. Flipping bit 63 equals adding
    2^63 modulo 2^64, so the same shift serves both streams."""
    if cols % 4 or r0 < 0:
        raise ValueError("cols must be a multiple of 4 and r0 non-negative")
    return (int(sr_seed) + (r0 * cols // 4) * GAMMA) % (1 << 64)


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
