"""Block scales in the block-scaled MMA layout, consumed by the hardware FP4 GEMM.

FP4Q_OUT_SCALES_MMA writes E4M3 (NVFP4) / UE8M0 (MXFP4) block scales in the 128 x 4 tile layout
of sm_100 block-scaled tensor-core MMA. Checks: the scales equal the oracle's row-major scales
rearranged into that layout as cuBLAS documents it; codes are unchanged; dequantize reads the
layout back; and the codes and scales, handed unchanged to torch's NVFP4 / MXFP4 scaled matmul
(cuBLASLt on the FP4 tensor cores), give the product of the decoded operands.
"""
import math

import numpy as np
import pytest

import oracle as O
import block_scaled_bit_rht16_b200 as fq
from block_scaled_bit_rht16_b200 import synth

from helpers import bf16_bits, host, ocfg, to_dev

pytestmark = pytest.mark.gpu

E2M1_VALUES = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6, -0.0, -0.5, -1, -1.5, -2, -3, -4, -6], np.float64)


def _to_blocked(scales_2d):
    """cuBLAS's block-scaling-factor layout restated with reshapes: 128 x 4 tiles, row-major over
    tiles; inside a tile the 128 rows are 4 groups of 32 and element (32i + j, c) lands at
    16j + 4i + c. (The hardware GEMM test below checks the layout independently.)"""
    r, c = scales_2d.shape
    t = scales_2d.reshape(r // 128, 128, c // 4, 4).transpose(0, 2, 1, 3)   # tiles
    return t.reshape(-1, 4, 32, 4).transpose(0, 2, 1, 3).reshape(-1)


def _cfgs():
    mask = fq.sign_mask_from_seed(synth.sign_seed(4))
    nv = fq.Config(grid=fq.FP4Q_GRID_E2M1, scale=fq.FP4Q_SCALE_E4M3_1x16_TENSOR, rht=1,
                   sign_mask=mask, mma_scales=True)
    mx = fq.Config(grid=fq.FP4Q_GRID_E2M1, scale=fq.FP4Q_SCALE_UE8M0_1x32, rht=1,
                   sign_mask=mask, mma_scales=True)
    return {"nvfp4": nv, "mxfp4": mx}


@pytest.mark.parametrize("kind", ["nvfp4", "mxfp4"])
@pytest.mark.parametrize("shape", [(128, 256), (384, 1024), (2048, 5120)])
def test_mma_scales_are_the_blocked_row_major_scales(kind, shape):
    import torch
    from dataclasses import replace
    cfg = _cfgs()[kind]
    rows, cols = shape
    x = synth.small(rows + cols, rows, cols, "laplace")
    q = fq.rht_quantize(cfg, to_dev(x))
    lin = fq.rht_quantize(replace(cfg, mma_scales=False), to_dev(x))
    ref = O.quantize(ocfg(cfg), x)
    np.testing.assert_array_equal(host(q.codes), ref["codes"])
    np.testing.assert_array_equal(host(lin.scales), ref["scales"])
    want = _to_blocked(np.ascontiguousarray(ref["scales"]))
    np.testing.assert_array_equal(host(q.scales).reshape(-1), want)
    # dequantize reads the same layout back
    d_mma = fq.dequantize(cfg, q.codes, q.scales, q.tensor_scale)
    d_lin = fq.dequantize(replace(cfg, mma_scales=False), lin.codes, lin.scales, lin.tensor_scale)
    np.testing.assert_array_equal(bf16_bits(d_mma), bf16_bits(d_lin))


def test_mma_layout_shape_rules():
    import torch
    cfg = _cfgs()["nvfp4"]
    x = to_dev(synth.small(5, 100, 256, "normal"))
    with pytest.raises(fq.Fp4qError):
        fq.rht_quantize(cfg, x)          # rows not a multiple of 128
    x = to_dev(synth.small(6, 128, 32, "normal"))
    with pytest.raises(fq.Fp4qError):
        fq.rht_quantize(cfg, x)          # 2 scale columns, not a multiple of 4
    from dataclasses import replace
    with pytest.raises(fq.Fp4qError):
        fq.rht_quantize(replace(cfg, scale=fq.FP4Q_SCALE_FP32_1x16), to_dev(synth.small(7, 128, 64)))


def _decoded(codes, block_scale, block):
    """Exact decoded operand: E2M1 value of every nibble times its block scale (FP64)."""
    c = codes.astype(np.int64)
    nib = np.stack([c & 0xF, c >> 4], axis=-1).reshape(codes.shape[0], -1)
    return E2M1_VALUES[nib] * np.repeat(block_scale, block, axis=1)


@pytest.mark.parametrize("kind", ["nvfp4", "mxfp4"])
def test_hardware_fp4_gemm_consumes_codes_and_scales(kind):
    import torch
    import torch.nn.functional as F
    from dataclasses import replace
    cfg = _cfgs()[kind]
    M, N, K = 1024, 512, 2048
    a_bits = synth.small(41, M, K, "t4")
    b_bits = synth.small(42, N, K, "normal", 0.02)
    qa, qb = fq.rht_quantize(cfg, to_dev(a_bits)), fq.rht_quantize(cfg, to_dev(b_bits))
    # exact operands from the row-major scales of the same quantization
    la = fq.rht_quantize(replace(cfg, mma_scales=False), to_dev(a_bits))
    lb = fq.rht_quantize(replace(cfg, mma_scales=False), to_dev(b_bits))
    if kind == "nvfp4":
        sa = torch.from_numpy(host(la.scales)).view(torch.float8_e4m3fn).double().numpy()
        sb = torch.from_numpy(host(lb.scales)).view(torch.float8_e4m3fn).double().numpy()
        block, alpha = 16, float(host(qa.tensor_scale)[0]) * float(host(qb.tensor_scale)[0])
        recipe, sdt = F.ScalingType.BlockWise1x16, torch.float8_e4m3fn
    else:
        sa = np.ldexp(1.0, host(la.scales).astype(np.int64) - 127)
        sb = np.ldexp(1.0, host(lb.scales).astype(np.int64) - 127)
        block, alpha = 32, 1.0
        recipe, sdt = F.ScalingType.BlockWise1x32, torch.float8_e8m0fnu
    ref = (_decoded(host(la.codes), sa, block) @ _decoded(host(lb.codes), sb, block).T) * alpha

    mat_a = qa.codes.view(torch.float4_e2m1fn_x2)
    mat_b = qb.codes.view(torch.float4_e2m1fn_x2).t()
    scale_a = qa.scales.view(sdt).reshape(M, K // block)
    scale_b = qb.scales.view(sdt).reshape(K // block, N)
    if kind == "nvfp4":
        out = F.scaled_mm(mat_a, mat_b, [scale_a, qa.tensor_scale],
                          [recipe, F.ScalingType.TensorWise], [scale_b, qb.tensor_scale],
                          [recipe, F.ScalingType.TensorWise],
                          swizzle_a=[F.SwizzleType.SWIZZLE_32_4_4],
                          swizzle_b=[F.SwizzleType.SWIZZLE_32_4_4], output_dtype=torch.bfloat16)
    else:
        out = F.scaled_mm(mat_a, mat_b, [scale_a], [recipe], [scale_b], [recipe],
                          swizzle_a=[F.SwizzleType.SWIZZLE_32_4_4],
                          swizzle_b=[F.SwizzleType.SWIZZLE_32_4_4], output_dtype=torch.bfloat16)
    got = out.double().cpu().numpy()
    sqnr = 10 * math.log10(float((ref ** 2).sum()) / float(((got - ref) ** 2).sum()))
    print("fp4 gemm %s: agreement with the FP64 product of the decoded operands %.1f dB" % (kind, sqnr))
    # bf16 output rounding alone allows ~50 dB; a misplaced scale would give ~0 dB
    assert sqnr > 40.0
