"""GPU parity at the full sizes of the five workloads, in the launch configuration the benchmark
times, compared with the oracle over the whole tensors (the oracle runs in row chunks on a
thread pool), every output between guard bands that must come back untouched.

  1  activation [512, 2048] with outlier columns: E2M1 and E1M2, with and without RHT16,
     codes + scales + dequant + statistics
  2  X, W [8192, 2048] each, UFP4 fwd_y, one launch over the stacked [16384, 2048]
  3  dY [8192, 8192], dual orientation with stochastic rounding: every row and every column
  4  [16384, 5120] Laplace: NVFP4, NVINT4, MXFP4, IF4 with the tensor scale computed on device,
     codes and scales, then the statistics the format comparison reports (MSE, IF4's FP4
     share) through the library against the oracle's
  5  MoE [64 x 2048, 7168] and dense [32768, 8192]: UFP4 and the E2M1 baseline
"""
import numpy as np
import pytest
import torch

import oracle as O
import block_scaled_bit_rht16_b200 as fq
from block_scaled_bit_rht16_b200 import synth
from helpers import (Canaries, bf16_bits, guarded_dual, guarded_quantized, host, ocfg, oracle_rows,
                     to_dev)
from test_parity_gpu import compare_stats

pytestmark = pytest.mark.gpu


def _quantize_guarded(cfg, bits):
    x = to_dev(bits)
    assert x.data_ptr() % 32 == 0      # the benchmark's launch: 256-bit loads
    guard = Canaries()
    out = fq.rht_quantize(cfg, x, out=guarded_quantized(cfg, bits.shape[0], bits.shape[1], guard))
    guard.check()
    del x
    return out


def _check_whole(cfg, bits, out, tensor_scale=None):
    ref = oracle_rows(ocfg(cfg), bits, tensor_scale=tensor_scale)
    codes, scales = host(out.codes), host(out.scales)
    bad = np.nonzero((codes != ref["codes"]).any(axis=1))[0]
    assert bad.size == 0, "codes differ in %d rows, first %s" % (bad.size, bad[:8].tolist())
    bad = np.nonzero((scales != ref["scales"]).any(axis=1))[0]
    assert bad.size == 0, "scales differ in %d rows, first %s" % (bad.size, bad[:8].tolist())


def test_outlier_activation_512x2048():
    x = synth.outlier_activation()
    mask = fq.sign_mask_from_seed(synth.sign_seed(1))
    sq = {}
    for grid in (fq.FP4Q_GRID_E2M1, fq.FP4Q_GRID_E1M2):
        for rht in (0, 1):
            cfg = fq.Config(grid=grid, rht=rht, sign_mask=mask, dequant=True, stats=True)
            out = _quantize_guarded(cfg, x)
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
    out = _quantize_guarded(cfg, bits)
    _check_whole(cfg, bits, out)


def test_backward_dy_8192x8192_dual_orientation():
    dy = synth.backward_dy()
    M, N = dy.shape
    mask = fq.sign_mask_from_seed(synth.sign_seed(3))
    rc = fq.recipe("ufp4", "bwd_dx", "dy", sign_mask=mask, sr_seed=synth.SR_SEED)
    cc = fq.recipe("ufp4", "bwd_dw", "dy", sign_mask=mask, sr_seed=synth.SR_SEED)
    guard = Canaries()
    out = fq.quantize_dual(rc, cc, to_dev(dy), out=guarded_dual(M, N, guard))
    guard.check()
    r = oracle_rows(ocfg(rc), dy)
    np.testing.assert_array_equal(host(out.codes_row), r["codes"])
    np.testing.assert_array_equal(host(out.scales_row), r["scales"])
    del r
    c = oracle_rows(ocfg(cc), np.ascontiguousarray(dy.T))
    np.testing.assert_array_equal(host(out.codes_col), c["codes"])
    np.testing.assert_array_equal(host(out.scales_col), c["scales"])


KINDS = {"nvfp4": (fq.FP4Q_GRID_E2M1, fq.FP4Q_SCALE_E4M3_1x16_TENSOR, 6.0),
         "nvint4": (fq.FP4Q_GRID_INT4, fq.FP4Q_SCALE_E4M3_1x16_TENSOR, 7.0),
         "mxfp4": (fq.FP4Q_GRID_E2M1, fq.FP4Q_SCALE_UE8M0_1x32, None),
         "if4": (fq.FP4Q_GRID_IF4, fq.FP4Q_SCALE_E4M3_1x16_TENSOR, 6.0)}


def _laplace_cfg(kind, stats=False):
    grid, scale, _ = KINDS[kind]
    return fq.Config(grid=grid, scale=scale, sign_mask=fq.sign_mask_from_seed(synth.sign_seed(4)),
                     stats=stats)


def _laplace_tensor_scale(kind, cfg, x):
    qmax = KINDS[kind][2]
    if qmax is None:
        return None
    A = O.tensor_amax(ocfg(cfg), x)
    return np.float32(np.float32(A) / np.float32(qmax * 448))


@pytest.mark.parametrize("kind", ["nvfp4", "nvint4", "mxfp4", "if4"])
def test_laplace_16384x5120_formats(kind):
    x = synth.laplace_format_tensor()
    cfg = _laplace_cfg(kind)
    out = _quantize_guarded(cfg, x)
    ts = _laplace_tensor_scale(kind, cfg, x)
    if ts is not None:
        assert host(out.tensor_scale)[0] == ts
    _check_whole(cfg, x, out, tensor_scale=ts)


@pytest.mark.parametrize("kind", ["nvfp4", "nvint4", "mxfp4", "if4"])
def test_laplace_16384x5120_format_statistics(kind):
    # the format comparison's figures (per-format MSE, IF4's share of FP4 blocks) produced by
    # the library's statistics output, against the oracle's over the same tensor
    x = synth.laplace_format_tensor()
    cfg = _laplace_cfg(kind, stats=True)
    out = _quantize_guarded(cfg, x)
    g = fq.stats(out.workspace)
    ts = _laplace_tensor_scale(kind, cfg, x)
    ref = oracle_rows(ocfg(cfg), x, tensor_scale=ts, stats=True)
    np.testing.assert_array_equal(host(out.codes), ref["codes"])
    raw = ref["stats_raw"]
    compare_stats(g, O.finalize_stats(raw), raw)
    assert g["n"] == x.size
    assert g["nmse"] == pytest.approx(raw[O.ST_SUM_ERR2] / raw[O.ST_SUM_Y2], rel=1e-5)
    if kind == "if4":
        assert 0.0 < g["if4_fp4_fraction"] < 1.0
    print("%s: nmse %.6e mse %.6e sqnr %.3f dB if4_fp4_fraction %.4f"
          % (kind, g["nmse"], g["mse"], g["sqnr_db"], g["if4_fp4_fraction"]))


@pytest.mark.parametrize("recipe", ["ufp4", "e2m1"])
def test_moe_experts_and_dense_layer(recipe):
    mask = fq.sign_mask_from_seed(synth.sign_seed(5))
    cfg = fq.recipe(recipe, "fwd_y", "x", sign_mask=mask)
    moe = np.concatenate([synth.moe_expert(e) for e in range(64)], axis=0)
    out = _quantize_guarded(cfg, moe)
    _check_whole(cfg, moe, out)
    del out, moe
    torch.cuda.empty_cache()
    dense = synth.dense_layer_rows(0, 32768)
    out = _quantize_guarded(cfg, dense)
    _check_whole(cfg, dense, out)
