"""The allocation-free quantize entry point, for callers that cannot allocate device memory
(plugin boundaries that pass only input/output buffers, frameworks that own all device memory,
work where cudaMalloc is off limits). It keeps the scratch of the device-side E4M3 tensor scale
in a static array inside the library; this test calls it through the C ABI and checks it against
the entry point that takes a caller-provided workspace, on two calls in a row whose tensors have
very different amaxes (so scratch left over from the first call would change the second's
result). Named to be collected last."""
import ctypes

import numpy as np
import pytest
import torch

import block_scaled_bit_rht16_b200 as fq
from block_scaled_bit_rht16_b200 import _lib, synth
from helpers import bf16_bits, host, to_dev

pytestmark = pytest.mark.gpu


def _noalloc(cfg, x, codes, scales, ts, dequant=None):
    c = cfg.c()
    ld = x.stride(0)
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    return _lib.load().fp4q_rht_quantize_noalloc(ctypes.byref(c), p(x), x.shape[0], x.shape[1], ld,
                                                 p(codes), p(scales), p(ts), 0, p(dequant), s)


@pytest.mark.parametrize("grid", [fq.FP4Q_GRID_E2M1, fq.FP4Q_GRID_IF4, fq.FP4Q_GRID_INT4])
def test_noalloc_matches_workspace_entry_point_twice(grid):
    cfg = fq.Config(grid=grid, scale=fq.FP4Q_SCALE_E4M3_1x16_TENSOR, sign_mask=0x3C3C, dequant=True)
    inputs = [synth.small(5, 300, 1024, "laplace", 50.0), synth.small(6, 300, 1024, "normal", 0.01)]
    for bits in inputs:                                  # two calls in a row
        x = to_dev(bits)
        ref = fq.rht_quantize(cfg, x)                    # caller-provided workspace
        codes = torch.empty_like(ref.codes)
        scales = torch.empty_like(ref.scales)
        ts = torch.full((1,), -1.0, dtype=torch.float32, device="cuda")
        deq = torch.empty_like(ref.dequant)
        assert _noalloc(cfg, x, codes, scales, ts, deq) == 0
        torch.cuda.synchronize()
        assert host(ts)[0] == host(ref.tensor_scale)[0]
        np.testing.assert_array_equal(host(codes), host(ref.codes))
        np.testing.assert_array_equal(host(scales), host(ref.scales))
        np.testing.assert_array_equal(bf16_bits(deq), bf16_bits(ref.dequant))


@pytest.mark.parametrize("cfg", [
    fq.Config(grid=fq.FP4Q_GRID_E1M2, round=fq.FP4Q_ROUND_SR, sign_mask=0x0FF0, sr_seed=0x5A5A0003),
    fq.Config(grid=fq.FP4Q_GRID_E2M1, scale=fq.FP4Q_SCALE_UE8M0_1x32, sign_mask=0x1234, dequant=True)],
    ids=["fp32-sr", "ue8m0-rtne"])
def test_noalloc_configurations_without_scratch(cfg):
    # FP32 and UE8M0 scales need no scratch at all: the entry point passes no workspace and must
    # still give the workspace entry point's results, stochastic rounding included
    for bits in [synth.small(7, 130, 512, "t4"), synth.small(8, 64, 1024, "normal", 1e-3)]:
        x = to_dev(bits)
        ref = fq.rht_quantize(cfg, x)
        codes, scales = torch.empty_like(ref.codes), torch.empty_like(ref.scales)
        deq = torch.empty_like(ref.dequant) if cfg.dequant else None
        assert _noalloc(cfg, x, codes, scales, None, deq) == 0
        torch.cuda.synchronize()
        np.testing.assert_array_equal(host(codes), host(ref.codes))
        np.testing.assert_array_equal(host(scales), host(ref.scales))
        if cfg.dequant:
            np.testing.assert_array_equal(bf16_bits(deq), bf16_bits(ref.dequant))


def test_noalloc_rejects_statistics():
    cfg = fq.Config(stats=True)
    x = torch.zeros((16, 64), dtype=torch.bfloat16, device="cuda")
    codes = torch.empty((16, 32), dtype=torch.uint8, device="cuda")
    scales = torch.empty((16, 4), dtype=torch.float32, device="cuda")
    assert _noalloc(cfg, x, codes, scales, None) == _lib.FP4Q_ERR_WORKSPACE
