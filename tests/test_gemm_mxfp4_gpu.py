"""The library's own MXFP4 GEMM on the 5th-generation tensor cores (fp4q_gemm_mxfp4), fed the
quantizer's E2M1 codes and MMA-layout UE8M0 block scales unchanged: checked against the FP64
product of the decoded operands, against cuBLASLt's MXFP4 GEMM on the same inputs, and timed
beside it ("AMD全新研究揭示：FP4训练不稳定性源于结构误差而非随机性不足": MXFP4 = 32-element blocks
with one shared power-of-two scale)."""
import math

import numpy as np
import pytest

import block_scaled_bit_rht16_b200 as fq
from block_scaled_bit_rht16_b200 import synth
from helpers import Canaries, host, to_dev

pytestmark = pytest.mark.gpu

E2M1_VALUES = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6, -0.0, -0.5, -1, -1.5, -2, -3, -4, -6], np.float64)


def _cfg(mma=True):
    return fq.Config(grid=fq.FP4Q_GRID_E2M1, scale=fq.FP4Q_SCALE_UE8M0_1x32, rht=1,
                     sign_mask=fq.sign_mask_from_seed(synth.sign_seed(2)), mma_scales=mma)


def _decoded(codes, scales_ue8m0):
    c = codes.astype(np.int64)
    nib = np.stack([c & 0xF, c >> 4], axis=-1).reshape(codes.shape[0], -1)
    s = np.ldexp(1.0, scales_ue8m0.astype(np.int64) - 127)
    return E2M1_VALUES[nib] * np.repeat(s, 32, axis=1)


def _sqnr(ref, got):
    return 10 * math.log10(float((ref ** 2).sum()) / max(float(((got - ref) ** 2).sum()), 1e-300))


@pytest.mark.parametrize("shape", [(128, 128, 256), (256, 384, 768), (1024, 512, 2048), (128, 768, 4096),
                                   (4096, 1280, 512), (4096, 1152, 256)])   # up to 288 tiles
def test_mxfp4_gemm_matches_the_decoded_product(shape):
    import torch
    from dataclasses import replace
    M, N, K = shape
    a_bits = synth.small(71 + M, M, K, "t4")
    b_bits = synth.small(72 + N, N, K, "normal", 0.02)
    cfg = _cfg()
    qa, qb = fq.rht_quantize(cfg, to_dev(a_bits)), fq.rht_quantize(cfg, to_dev(b_bits))
    la = fq.rht_quantize(replace(cfg, mma_scales=False), to_dev(a_bits))
    lb = fq.rht_quantize(replace(cfg, mma_scales=False), to_dev(b_bits))
    ref = _decoded(host(la.codes), host(la.scales)) @ _decoded(host(lb.codes), host(lb.scales)).T
    guard = Canaries()
    out = guard.empty((M, N), torch.bfloat16)
    fq.gemm_mxfp4(qa, qb, out=out)
    guard.check()
    sq = _sqnr(ref, out.double().cpu().numpy())
    print("mxfp4 gemm %dx%dx%d: %.1f dB against the FP64 product of the decoded operands" % (M, N, K, sq))
    # bf16 output rounding alone allows ~50 dB; a misplaced scale or tile gives ~0 dB
    assert sq > 40.0


def test_mxfp4_gemm_agrees_with_cublaslt_and_timing():
    import torch
    import torch.nn.functional as F
    M, N, K = 4096, 4096, 8192
    a_bits = synth.small(81, M, K, "t4")
    b_bits = synth.small(82, N, K, "normal", 0.02)
    cfg = _cfg()
    qa, qb = fq.rht_quantize(cfg, to_dev(a_bits)), fq.rht_quantize(cfg, to_dev(b_bits))
    ours = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    sdt = torch.float8_e8m0fnu

    def lib():
        fq.gemm_mxfp4(qa, qb, out=ours)

    def cublaslt():
        return F.scaled_mm(qa.codes.view(torch.float4_e2m1fn_x2), qb.codes.view(torch.float4_e2m1fn_x2).t(),
                           [qa.scales.view(sdt).reshape(M, K // 32)], [F.ScalingType.BlockWise1x32],
                           [qb.scales.view(sdt).reshape(K // 32, N)], [F.ScalingType.BlockWise1x32],
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
    print("mxfp4 gemm %dx%dx%d: library %.3f ms (%.0f TFLOP/s), cuBLASLt %.3f ms (%.0f TFLOP/s); "
          "outputs agree to %.1f dB" % (M, N, K, times["library"], tf["library"], times["cublaslt"],
                                         tf["cublaslt"], sq))
    # both accumulate exact products in FP32 (in different orders) and round to bf16
    assert sq > 45.0


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4"])
def test_gemm_into_a_row_pitched_output(fmt):
    # out with ldo = N + 64: the result equals the contiguous one, the pad columns stay untouched
    import torch
    M, N, K = 512, 512, 1024
    scale = fq.FP4Q_SCALE_E4M3_1x16_TENSOR if fmt == "nvfp4" else fq.FP4Q_SCALE_UE8M0_1x32
    cfg = fq.Config(grid=fq.FP4Q_GRID_E2M1, scale=scale, rht=1,
                    sign_mask=fq.sign_mask_from_seed(synth.sign_seed(2)), mma_scales=True)
    qa = fq.rht_quantize(cfg, to_dev(synth.small(91, M, K, "t4")))
    qb = fq.rht_quantize(cfg, to_dev(synth.small(92, N, K, "normal", 0.02)))
    gemm = fq.gemm_nvfp4 if fmt == "nvfp4" else fq.gemm_mxfp4
    ref = gemm(qa, qb)
    wide = torch.full((M, N + 64), -7.0, dtype=torch.bfloat16, device="cuda")
    gemm(qa, qb, out=wide[:, :N])
    torch.cuda.synchronize()
    assert torch.equal(wide[:, :N], ref)
    assert bool((wide[:, N:] == -7.0).all())
