"""The library's own NVFP4 GEMM on the 5th-generation tensor cores (fp4q_gemm_nvfp4), fed the
quantizer's E2M1 codes, MMA-layout E4M3 block scales and FP32 tensor scales unchanged: checked
against the FP64 product of the decoded operands, against cuBLASLt's NVFP4 GEMM on the same
inputs, and timed beside it ("低精度量化技术：IF4…", section 3.2: NVFP4's two-level scales are the
hardware path)."""
import math

import numpy as np
import pytest

import block_scaled_bit_rht16_b200 as fq
from block_scaled_bit_rht16_b200 import synth
from helpers import Canaries, host, to_dev

pytestmark = pytest.mark.gpu

E2M1_VALUES = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6, -0.0, -0.5, -1, -1.5, -2, -3, -4, -6], np.float64)


def _cfg(mma=True):
    return fq.Config(grid=fq.FP4Q_GRID_E2M1, scale=fq.FP4Q_SCALE_E4M3_1x16_TENSOR, rht=1,
                     sign_mask=fq.sign_mask_from_seed(synth.sign_seed(2)), mma_scales=mma)


def _decoded(codes, scales_e4m3, ts):
    import torch
    c = codes.astype(np.int64)
    nib = np.stack([c & 0xF, c >> 4], axis=-1).reshape(codes.shape[0], -1)
    s = torch.from_numpy(scales_e4m3).view(torch.float8_e4m3fn).double().numpy()
    return E2M1_VALUES[nib] * np.repeat(s, 16, axis=1) * ts


def _sqnr(ref, got):
    return 10 * math.log10(float((ref ** 2).sum()) / max(float(((got - ref) ** 2).sum()), 1e-300))


@pytest.mark.parametrize("shape", [(128, 128, 256), (256, 384, 768), (1024, 512, 2048), (128, 768, 4096),
                                   (4096, 1280, 512), (4096, 1152, 256)])   # more tiles than SMs
def test_gemm_matches_the_decoded_product(shape):
    import torch
    from dataclasses import replace
    M, N, K = shape
    a_bits = synth.small(51 + M, M, K, "t4")
    b_bits = synth.small(52 + N, N, K, "normal", 0.02)
    cfg = _cfg()
    qa, qb = fq.rht_quantize(cfg, to_dev(a_bits)), fq.rht_quantize(cfg, to_dev(b_bits))
    la = fq.rht_quantize(replace(cfg, mma_scales=False), to_dev(a_bits))
    lb = fq.rht_quantize(replace(cfg, mma_scales=False), to_dev(b_bits))
    ref = _decoded(host(la.codes), host(la.scales), float(host(la.tensor_scale)[0])) @ \
        _decoded(host(lb.codes), host(lb.scales), float(host(lb.tensor_scale)[0])).T
    guard = Canaries()
    out = guard.empty((M, N), torch.bfloat16)
    fq.gemm_nvfp4(qa, qb, out=out)
    guard.check()
    got = out.double().cpu().numpy()
    sq = _sqnr(ref, got)
    print("nvfp4 gemm %dx%dx%d: %.1f dB against the FP64 product of the decoded operands" % (M, N, K, sq))
    # bf16 output rounding alone allows ~50 dB; a misplaced scale or tile gives ~0 dB
    assert sq > 40.0


def test_gemm_agrees_with_cublaslt_and_timing():
    import torch
    import torch.nn.functional as F
    M, N, K = 4096, 4096, 8192
    a_bits = synth.small(61, M, K, "t4")
    b_bits = synth.small(62, N, K, "normal", 0.02)
    cfg = _cfg()
    qa, qb = fq.rht_quantize(cfg, to_dev(a_bits)), fq.rht_quantize(cfg, to_dev(b_bits))
    ours = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    sdt = torch.float8_e4m3fn

    def lib():
        fq.gemm_nvfp4(qa, qb, out=ours)

    def cublaslt():
        return F.scaled_mm(qa.codes.view(torch.float4_e2m1fn_x2), qb.codes.view(torch.float4_e2m1fn_x2).t(),
                           [qa.scales.view(sdt).reshape(M, K // 16), qa.tensor_scale],
                           [F.ScalingType.BlockWise1x16, F.ScalingType.TensorWise],
                           [qb.scales.view(sdt).reshape(K // 16, N), qb.tensor_scale],
                           [F.ScalingType.BlockWise1x16, F.ScalingType.TensorWise],
                           swizzle_a=[F.SwizzleType.SWIZZLE_32_4_4], swizzle_b=[F.SwizzleType.SWIZZLE_32_4_4],
                           output_dtype=torch.bfloat16)
    lib()
    theirs = cublaslt()
    torch.cuda.synchronize()
    sq = _sqnr(theirs.double().cpu().numpy(), ours.double().cpu().numpy())
    times = {}
    for name, fn in (("library", lib), ("cublaslt", cublaslt)):
        for _ in range(3):
            fn()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record()
        for _ in range(20):
            fn()
        b.record()
        torch.cuda.synchronize()
        times[name] = a.elapsed_time(b) / 20
    tf = {k: 2.0 * M * N * K / (v * 1e-3) / 1e12 for k, v in times.items()}
    print("nvfp4 gemm %dx%dx%d: library %.3f ms (%.0f TFLOP/s), cuBLASLt %.3f ms (%.0f TFLOP/s); "
          "outputs agree to %.1f dB" % (M, N, K, times["library"], tf["library"], times["cublaslt"],
                                         tf["cublaslt"], sq))
    # both accumulate exact products in FP32 (in different orders) and round to bf16
    assert sq > 45.0


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4"])
def test_half_tiles_of_the_last_round_equal_whole_tiles(fmt):
    # 4096 x 1280: 160 tiles of 128 x 256 on at most 148 CTAs, so the last round's tiles run as
    # 128 x 128 halves; the column blocks [0, 1024) and [1024, 1280) as GEMMs of their own (128
    # and 32 tiles) run as whole tiles. Each output element is the same sum in the same order.
    import torch
    M, N, K = 4096, 1280, 512
    scale = fq.FP4Q_SCALE_E4M3_1x16_TENSOR if fmt == "nvfp4" else fq.FP4Q_SCALE_UE8M0_1x32
    cfg = fq.Config(grid=fq.FP4Q_GRID_E2M1, scale=scale, rht=1,
                    sign_mask=fq.sign_mask_from_seed(synth.sign_seed(2)), mma_scales=True)
    gemm = fq.gemm_nvfp4 if fmt == "nvfp4" else fq.gemm_mxfp4
    qa = fq.rht_quantize(cfg, to_dev(synth.small(93, M, K, "t4")))
    b = to_dev(synth.small(94, N, K, "normal", 0.02))
    qb = fq.rht_quantize(cfg, b)
    whole = gemm(qa, qb)
    parts = []
    for c0, c1 in ((0, 1024), (1024, N)):
        # the rows of B quantized alone, with the whole B's tensor scale (NVFP4): the same codes
        # and block scales as those rows of qb
        q = fq.rht_quantize(cfg, b[c0:c1].contiguous(), tensor_scale=qb.tensor_scale,
                            tensor_scale_given=fmt == "nvfp4")
        parts.append(gemm(qa, q))
    torch.cuda.synchronize()
    assert torch.equal(whole[:, :1024], parts[0])
    assert torch.equal(whole[:, 1024:], parts[1])
