"""GPU parity at the full sizes of the five workloads, in the launch configuration the benchmark
times, compared with the oracle on sampled rows (and columns for the dual orientation).

  1  activation [512, 2048] with outlier columns: E2M1 and E1M2, with and without RHT16,
     codes + scales + dequant + statistics, compared whole (the oracle finishes in seconds)
  2  X, W [8192, 2048] each, UFP4 fwd_y, one launch over the stacked [16384, 2048]
  3  dY [8192, 8192], dual orientation with stochastic rounding
  4  [16384, 5120] Laplace: NVFP4, NVINT4, MXFP4, IF4 with the tensor scale computed on device
  5  MoE [64 x 2048, 7168] and dense [32768, 8192]: UFP4 and the E2M1 baseline
"""
import numpy as np
import pytest
import torch

import oracle as O
import block_scaled_bit_rht16_b200 as fq
from block_scaled_bit_rht16_b200 import synth
from helpers import bf16_bits, host, ocfg, to_dev
from test_parity_gpu import compare_stats

pytestmark = pytest.mark.gpu


def _sample_rows(n, k, seed):
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(n, size=min(k, n), replace=False).tolist()) | {0, n - 1}
    return sorted(rows)


def _check_rows(cfg, bits, out, rows, tensor_scale=None):
    oc = ocfg(cfg)
    codes, scales = host(out.codes), host(out.scales)
    for r in rows:
        ref = O.quantize(oc, np.ascontiguousarray(bits[r:r + 1]), row0=r, tensor_scale=tensor_scale)
        np.testing.assert_array_equal(codes[r], ref["codes"][0], err_msg="row %d" % r)
        np.testing.assert_array_equal(scales[r], ref["scales"][0], err_msg="row %d" % r)


def test_outlier_activation_512x2048():
    x = synth.outlier_activation()
    mask = fq.sign_mask_from_seed(synth.sign_seed(1))
    sq = {}
    for grid in (fq.FP4Q_GRID_E2M1, fq.FP4Q_GRID_E1M2):
        for rht in (0, 1):
            cfg = fq.Config(grid=grid, rht=rht, sign_mask=mask, dequant=True, stats=True)
            out = fq.rht_quantize(cfg, to_dev(x))
            g = fq.stats(out.workspace)
            ref = O.quantize(ocfg(cfg), x, dequant=True, stats=True)
            np.testing.assert_array_equal(host(out.codes), ref["codes"])
            np.testing.assert_array_equal(host(out.scales), ref["scales"])
            np.testing.assert_array_equal(bf16_bits(out.dequant), ref["dequant"])
            compare_stats(g, O.finalize_stats(ref["stats_raw"]), ref["stats_raw"])
            sq[grid, rht] = g["sqnr_db"]
    # the reversal the UFP4 pages describe (direction only)
    assert sq[fq.FP4Q_GRID_E1M2, 1] > sq[fq.FP4Q_GRID_E2M1, 1]
    assert sq[fq.FP4Q_GRID_E2M1, 0] >= sq[fq.FP4Q_GRID_E1M2, 0]


def test_dense_linear_operands_stacked_16384x2048():
    x, w = synth.dense_linear_operands()
    bits = np.concatenate([x, w], axis=0)
    mask = fq.sign_mask_from_seed(synth.sign_seed(2))
    cfg = fq.recipe("ufp4", "fwd_y", "x", sign_mask=mask)
    t = to_dev(bits)
    assert t.data_ptr() % 32 == 0      # the benchmark's launch: 256-bit loads
    out = fq.rht_quantize(cfg, t)
    torch.cuda.synchronize()
    _check_rows(cfg, bits, out, _sample_rows(bits.shape[0], 192, 2) + [8191, 8192])


def test_backward_dy_8192x8192_dual_orientation():
    dy = synth.backward_dy()
    mask = fq.sign_mask_from_seed(synth.sign_seed(3))
    rc = fq.recipe("ufp4", "bwd_dx", "dy", sign_mask=mask, sr_seed=synth.SR_SEED)
    cc = fq.recipe("ufp4", "bwd_dw", "dy", sign_mask=mask, sr_seed=synth.SR_SEED)
    out = fq.quantize_dual(rc, cc, to_dev(dy))
    torch.cuda.synchronize()
    cr, sr_ = host(out.codes_row), host(out.scales_row)
    for r in _sample_rows(dy.shape[0], 48, 3):
        ref = O.quantize(ocfg(rc), np.ascontiguousarray(dy[r:r + 1]), row0=r)
        np.testing.assert_array_equal(cr[r], ref["codes"][0])
        np.testing.assert_array_equal(sr_[r], ref["scales"][0])
    cc_, sc_ = host(out.codes_col), host(out.scales_col)
    for n in _sample_rows(dy.shape[1], 48, 4):
        col = np.ascontiguousarray(dy[:, n][None, :])
        ref = O.quantize(ocfg(cc), col, row0=n)
        np.testing.assert_array_equal(cc_[n], ref["codes"][0])
        np.testing.assert_array_equal(sc_[n], ref["scales"][0])


@pytest.mark.parametrize("kind", ["nvfp4", "nvint4", "mxfp4", "if4"])
def test_laplace_16384x5120_formats(kind):
    x = synth.laplace_format_tensor()
    mask = fq.sign_mask_from_seed(synth.sign_seed(4))
    grid = {"nvfp4": fq.FP4Q_GRID_E2M1, "nvint4": fq.FP4Q_GRID_INT4, "mxfp4": fq.FP4Q_GRID_E2M1,
            "if4": fq.FP4Q_GRID_IF4}[kind]
    scale = fq.FP4Q_SCALE_UE8M0_1x32 if kind == "mxfp4" else fq.FP4Q_SCALE_E4M3_1x16_TENSOR
    cfg = fq.Config(grid=grid, scale=scale, sign_mask=mask)
    out = fq.rht_quantize(cfg, to_dev(x))
    torch.cuda.synchronize()
    ts = None
    if scale == fq.FP4Q_SCALE_E4M3_1x16_TENSOR:
        A = O.tensor_amax(ocfg(cfg), x)
        qmax = 7.0 if kind == "nvint4" else 6.0
        ts = np.float32(np.float32(A) / np.float32(qmax * 448))
        assert host(out.tensor_scale)[0] == ts
    _check_rows(cfg, x, out, _sample_rows(x.shape[0], 96, 5), tensor_scale=ts)


@pytest.mark.parametrize("recipe", ["ufp4", "e2m1"])
def test_moe_experts_and_dense_layer(recipe):
    mask = fq.sign_mask_from_seed(synth.sign_seed(5))
    cfg = fq.recipe(recipe, "fwd_y", "x", sign_mask=mask)
    experts = [synth.moe_expert(e) for e in range(64)]
    moe = np.concatenate(experts, axis=0)
    del experts
    out = fq.rht_quantize(cfg, to_dev(moe))
    torch.cuda.synchronize()
    _check_rows(cfg, moe, out, _sample_rows(moe.shape[0], 96, 6))
    del out, moe
    dense = synth.dense_layer_rows(0, 32768)
    out = fq.rht_quantize(cfg, to_dev(dense))
    torch.cuda.synchronize()
    _check_rows(cfg, dense, out, _sample_rows(dense.shape[0], 64, 7))
