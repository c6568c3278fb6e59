"""The Python binding refuses buffers the library would misuse through a raw pointer (host
memory, a wrong element type, too few elements, a strided view) before any call into the
library, and a good call afterwards still matches the oracle."""
import numpy as np
import pytest
import torch

import oracle as O
import block_scaled_bit_rht16_b200 as fq
from block_scaled_bit_rht16_b200 import synth

from helpers import host, ocfg, to_dev

pytestmark = pytest.mark.gpu

E4M3 = fq.FP4Q_SCALE_E4M3_1x16_TENSOR


def _x(rows=64, cols=256):
    return to_dev(synth.small(3, rows, cols, "normal"))


def test_row_quantize_output_buffers_are_checked():
    cfg = fq.Config(sign_mask=0x0F0F)
    x = _x()
    good = fq.rht_quantize(cfg, x)
    bad_codes = fq.Quantized(good.codes[:32], good.scales, None, None, None)          # too short
    with pytest.raises(ValueError):
        fq.rht_quantize(cfg, x, out=bad_codes)
    bad_scales = fq.Quantized(good.codes, good.scales.view(torch.uint8), None, None, None)
    with pytest.raises(TypeError):
        fq.rht_quantize(cfg, x, out=bad_scales)                                        # FP32 expected
    host_codes = fq.Quantized(good.codes.cpu(), good.scales, None, None, None)
    with pytest.raises(TypeError):
        fq.rht_quantize(cfg, x, out=host_codes)
    strided = torch.empty((64, 256), dtype=torch.uint8, device="cuda")[:, ::2]
    with pytest.raises(ValueError):
        fq.rht_quantize(cfg, x, out=fq.Quantized(strided, good.scales, None, None, None))
    deq_cfg = fq.Config(sign_mask=0x0F0F, dequant=True)
    with pytest.raises(TypeError):
        fq.rht_quantize(deq_cfg, x, out=fq.Quantized(good.codes, good.scales, None, None, None))


def test_tensor_scales_and_offsets_are_checked():
    cfg = fq.Config(grid=fq.FP4Q_GRID_E2M1, scale=E4M3, sign_mask=0x0F0F)
    x = _x()
    with pytest.raises(TypeError):   # host memory
        fq.rht_quantize(cfg, x, tensor_scale=torch.ones(1), tensor_scale_given=True)
    with pytest.raises(TypeError):   # float64
        fq.rht_quantize(cfg, x, tensor_scale=torch.ones(1, dtype=torch.float64, device="cuda"),
                        tensor_scale_given=True)
    offs = torch.tensor([0, 20, 64], dtype=torch.int64)
    with pytest.raises(TypeError):   # offsets in host memory
        fq.rht_quantize_grouped(cfg, x, offs)
    with pytest.raises(TypeError):   # int32 offsets
        fq.rht_quantize_grouped(cfg, x, offs.to(torch.int32).cuda())
    with pytest.raises(ValueError):  # one tensor scale for two groups
        fq.rht_quantize_grouped(cfg, x, offs.cuda(), tensor_scales=torch.ones(1, device="cuda"),
                                tensor_scales_given=True)
    q = fq.rht_quantize(cfg, x)
    with pytest.raises(TypeError):
        fq.dequantize(cfg, q.codes, q.scales, q.tensor_scale.cpu())
    with pytest.raises(TypeError):
        fq.dequantize(cfg, q.codes, q.scales, None)


def test_dual_outputs_are_checked_and_a_good_call_still_matches_the_oracle():
    rc = fq.Config(round=fq.FP4Q_ROUND_SR, sr_seed=9, sign_mask=0x1111)
    cc = fq.Config(round=fq.FP4Q_ROUND_SR, sr_seed=9, sr_stream=1, sign_mask=0x1111)
    bits = synth.small(8, 64, 128, "normal")
    dy = to_dev(bits)
    good = fq.quantize_dual(rc, cc, dy)
    short = fq.Dual(good.codes_row, good.scales_row, good.codes_col[:10], good.scales_col)
    with pytest.raises(ValueError):
        fq.quantize_dual(rc, cc, dy, out=short)
    torch.cuda.synchronize()
    ref = O.quantize(ocfg(rc), bits)
    np.testing.assert_array_equal(host(good.codes_row), ref["codes"])
    np.testing.assert_array_equal(host(good.scales_row), ref["scales"])
    col = O.quantize(ocfg(cc), np.ascontiguousarray(bits.T))
    np.testing.assert_array_equal(host(good.codes_col), col["codes"])
    assert fq.device_status() == 0
