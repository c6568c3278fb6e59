"""Grouped quantization (MoE experts with variable token counts) against the oracle run once per
group: each group is its own tensor, with its own E4M3 tensor scale, and SR/row indices global."""
import numpy as np
import pytest
import torch

import oracle as O
import block_scaled_bit_rht16_b200 as fq
from block_scaled_bit_rht16_b200 import synth

from helpers import host, ocfg, to_dev

pytestmark = pytest.mark.gpu

E2M1, E1M2, INT4, IF4 = fq.FP4Q_GRID_E2M1, fq.FP4Q_GRID_E1M2, fq.FP4Q_GRID_INT4, fq.FP4Q_GRID_IF4
E4M3, FP32 = fq.FP4Q_SCALE_E4M3_1x16_TENSOR, fq.FP4Q_SCALE_FP32_1x16
MASK = 0x3C5A


def _offsets(sizes):
    return np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)


def _oracle_grouped(cfg, x, offs, given=None):
    codes, scales, ts = [], [], []
    for g in range(len(offs) - 1):
        r0, r1 = int(offs[g]), int(offs[g + 1])
        if r1 == r0:
            ts.append(np.float32(0.0) if given is None else given[g])
            continue
        out = O.quantize(ocfg(cfg), np.ascontiguousarray(x[r0:r1]), row0=r0,
                         tensor_scale=None if given is None else given[g])
        codes.append(out["codes"])
        scales.append(out["scales"])
        ts.append(np.float32(out["tensor_scale"]) if given is None else given[g])
    return np.concatenate(codes), np.concatenate(scales), np.array(ts, np.float32)


# experts with scales of their own (sigma_e log-uniform, as in the MoE workload), including empty
# experts, a single-row expert, and empty first and last experts
SIZES = [0, 37, 1, 0, 130, 64, 5, 211, 0]


def _moe_rows(sizes, cols, seed):
    rng = np.random.default_rng(seed)
    parts = [synth.small(seed + i, n, cols, "normal", float(10 ** rng.uniform(-1, 1)))
             for i, n in enumerate(sizes) if n]
    return np.concatenate(parts)


@pytest.mark.parametrize("grid", [E2M1, E1M2, INT4, IF4])
@pytest.mark.parametrize("rht", [0, 1])
def test_grouped_e4m3_matches_per_group_oracle(grid, rht):
    cols = 1056
    x = _moe_rows(SIZES, cols, 11 + grid)
    offs = _offsets(SIZES)
    cfg = fq.Config(grid=grid, scale=E4M3, rht=rht, sign_mask=MASK if rht else 0)
    q = fq.rht_quantize_grouped(cfg, to_dev(x), torch.from_numpy(offs).cuda())
    codes, scales, ts = _oracle_grouped(cfg, x, offs)
    np.testing.assert_array_equal(host(q.codes), codes)
    np.testing.assert_array_equal(host(q.scales), scales)
    np.testing.assert_array_equal(host(q.tensor_scale), ts)
    # the same groups with the tensor scales given (stale ones: halved)
    given = (ts * np.float32(0.5)).astype(np.float32)
    q2 = fq.rht_quantize_grouped(cfg, to_dev(x), torch.from_numpy(offs).cuda(),
                                 tensor_scales=torch.from_numpy(given).cuda(), tensor_scales_given=True)
    codes2, scales2, _ = _oracle_grouped(cfg, x, offs, given=given)
    np.testing.assert_array_equal(host(q2.codes), codes2)
    np.testing.assert_array_equal(host(q2.scales), scales2)


def test_grouped_large_many_iterations_and_mma_layout():
    # 64 experts of 2048 +- tokens, hidden 7168 / 4: many persistent-grid iterations per thread
    rng = np.random.default_rng(5)
    sizes = [int(n) for n in rng.integers(1, 33, size=64) * 128]   # multiples of 128 rows
    x = _moe_rows(sizes, 1792, 77)
    offs = _offsets(sizes)
    cfg = fq.Config(grid=E2M1, scale=E4M3, rht=1, sign_mask=MASK)
    q = fq.rht_quantize_grouped(cfg, to_dev(x), torch.from_numpy(offs).cuda())
    ts = host(q.tensor_scale)
    for g in (0, 17, 63):   # sampled experts against the oracle
        r0, r1 = int(offs[g]), int(offs[g + 1])
        out = O.quantize(ocfg(cfg), np.ascontiguousarray(x[r0:r1]), row0=r0)
        assert ts[g] == np.float32(out["tensor_scale"])
        np.testing.assert_array_equal(host(q.codes)[r0:r1], out["codes"])
        np.testing.assert_array_equal(host(q.scales)[r0:r1], out["scales"])
    # scales in the block-scaled MMA layout: the same bytes, rearranged by the slot function
    from dataclasses import replace
    qm = fq.rht_quantize_grouped(replace(cfg, mma_scales=True), to_dev(x), torch.from_numpy(offs).cuda())
    np.testing.assert_array_equal(host(qm.codes), host(q.codes))
    lin = host(q.scales)
    r, c = lin.shape
    t = lin.reshape(r // 128, 128, c // 4, 4).transpose(0, 2, 1, 3)
    np.testing.assert_array_equal(host(qm.scales).reshape(-1),
                                  t.reshape(-1, 4, 32, 4).transpose(0, 2, 1, 3).reshape(-1))


@pytest.mark.parametrize("rnd", [fq.FP4Q_ROUND_RTNE, fq.FP4Q_ROUND_SR])
def test_grouped_fp32_is_one_flat_call(rnd):
    x = _moe_rows(SIZES, 512, 3)
    offs = _offsets(SIZES)
    cfg = fq.Config(grid=E1M2, scale=FP32, round=rnd, rht=1, sign_mask=MASK, sr_seed=5)
    q = fq.rht_quantize_grouped(cfg, to_dev(x), torch.from_numpy(offs).cuda())
    flat = fq.rht_quantize(cfg, to_dev(x))
    np.testing.assert_array_equal(host(q.codes), host(flat.codes))
    np.testing.assert_array_equal(host(q.scales), host(flat.scales))
    ref = O.quantize(ocfg(cfg), x)
    np.testing.assert_array_equal(host(q.codes), ref["codes"])
