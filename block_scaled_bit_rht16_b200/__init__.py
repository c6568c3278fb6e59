"""Fused 16-point random Hadamard rotation + block-scaled 4-bit quantization for NVIDIA B200.

Thin Python binding of libfp4q (include/fp4q.h): argument marshalling only. Every step of the
quantizer runs in the library's sm_100a kernels; torch supplies device memory and streams.
Tensors are torch CUDA tensors; bf16 inputs are 2-D with a unit column stride (the row pitch
is passed as ``ld``).

Quantization recipes follow the UFP4 explainer "当你的 GPU 学不会算账"
(zhichai.net/topic/178208020), recipe table of section "UFP4：换一把尺子": UFP4 = E1M2, 1x16
blocks, FP32 single-level scale, rotation on fwd_y, bwd_dx and bwd_dw, stochastic rounding on
dY only; the E2M1 baseline = E2M1, same blocks and scale, rotation only on bwd_dw, stochastic
rounding on dY.
"""
import ctypes
from dataclasses import dataclass, replace

from . import _lib
from ._lib import (FP4Q_GRID_E1M2, FP4Q_GRID_E2M1, FP4Q_GRID_IF4, FP4Q_GRID_INT4,  # noqa: F401
                   FP4Q_OUT_CODES, FP4Q_OUT_DEQUANT, FP4Q_OUT_SCALES_MMA, FP4Q_OUT_STATS, FP4Q_ROUND_RTNE,
                   FP4Q_ROUND_SR, FP4Q_SCALE_E4M3_1x16_TENSOR, FP4Q_SCALE_FP32_1x16,
                   FP4Q_SCALE_UE8M0_1x32, Fp4qError)



@dataclass(frozen=True)
class Config:
    """Mirror of fp4q_config."""
    grid: int = FP4Q_GRID_E1M2
    scale: int = FP4Q_SCALE_FP32_1x16
    round: int = FP4Q_ROUND_RTNE
    rht: int = 1
    sign_mask: int = 0
    sr_stream: int = 0
    sr_seed: int = 0
    dequant: bool = False
    stats: bool = False
    e2m1_max: int = 0   # 4, 3, 2: range-restricted E2M1 (grid E2M1, FP32 1x16 scale)
    mma_scales: bool = False   # E4M3 / UE8M0 scales in the block-scaled MMA tile layout

    def c(self) -> _lib.fp4q_config:
        outputs = FP4Q_OUT_CODES | (FP4Q_OUT_DEQUANT if self.dequant else 0) | \
            (FP4Q_OUT_STATS if self.stats else 0) | (FP4Q_OUT_SCALES_MMA if self.mma_scales else 0)
        return _lib.fp4q_config(self.grid, self.scale, self.round, self.rht, self.sign_mask,
                                self.sr_stream, self.sr_seed & 0xFFFFFFFFFFFFFFFF, outputs,
                                self.e2m1_max)

    @property
    def block(self) -> int:
        return 32 if self.scale == FP4Q_SCALE_UE8M0_1x32 else 16


def recipe(name: str, path: str, operand: str, sign_mask: int = 0, sr_seed: int = 0) -> Config:
    """Config of one GEMM operand under a recipe.

    name: "ufp4" | "e2m1"; path: "fwd_y" | "bwd_dx" | "bwd_dw";
    operand: "x" | "w" | "dy" (the tensor being quantized along that GEMM's reduction axis).
    """
    if name not in ("ufp4", "e2m1") or path not in ("fwd_y", "bwd_dx", "bwd_dw"):
        raise ValueError("unknown recipe or path")
    grid = FP4Q_GRID_E1M2 if name == "ufp4" else FP4Q_GRID_E2M1
    rht = 1 if (name == "ufp4" or path == "bwd_dw") else 0
    sr = operand == "dy"
    stream = 1 if (sr and path == "bwd_dw") else 0
    return Config(grid=grid, rht=rht, sign_mask=sign_mask if rht else 0,
                  round=FP4Q_ROUND_SR if sr else FP4Q_ROUND_RTNE,
                  sr_seed=sr_seed if sr else 0, sr_stream=stream)


def _torch():
    import torch
    return torch


def _stream_ptr(stream, device=None):
    """The stream handle: `stream`, else torch's current stream on `device`."""
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check_input(x, name="x"):
    torch = _torch()
    if not (isinstance(x, torch.Tensor) and x.is_cuda and x.dtype == torch.bfloat16 and x.dim() == 2):
        raise TypeError("%s must be a 2-D bfloat16 CUDA tensor" % name)
    if x.stride(1) != 1 and x.numel() > 0:
        raise ValueError("%s must have unit column stride" % name)
    ld = x.stride(0) if (x.shape[0] > 1 and x.numel() > 0) else x.shape[1]
    return x.shape[0], x.shape[1], ld


def _check_buf(t, name, dtype, numel, device):
    """A buffer the library reads or writes through a raw pointer: a contiguous CUDA tensor of
    `dtype` on `device` with at least `numel` elements. Checked here because the C ABI cannot
    tell a host pointer or a short buffer from a good one."""
    torch = _torch()
    if not (isinstance(t, torch.Tensor) and t.is_cuda):
        raise TypeError("%s must be a CUDA tensor" % name)
    if t.device != device:
        raise ValueError("%s is on %s but the input is on %s" % (name, t.device, device))
    if t.dtype != dtype:
        raise TypeError("%s must be %s, not %s" % (name, dtype, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if t.numel() < numel:
        raise ValueError("%s holds %d elements, %d needed" % (name, t.numel(), numel))


def _scale_dtype(cfg):
    torch = _torch()
    return torch.float32 if cfg.scale == FP4Q_SCALE_FP32_1x16 else torch.uint8


def _check_quantized(cfg, out, rows, cols, device, dequant=False):
    """The code and scale buffers (and the dequant buffer when requested) of a row quantizer."""
    torch = _torch()
    _check_buf(out.codes, "codes", torch.uint8, rows * (cols // 2), device)
    _check_buf(out.scales, "scales", _scale_dtype(cfg), rows * (cols // cfg.block), device)
    if dequant:
        _check_buf(out.dequant, "dequant", torch.bfloat16, rows * cols, device)


def sign_mask_from_seed(seed: int) -> int:
    return int(_lib.load().fp4q_sign_mask_from_seed(seed & 0xFFFFFFFFFFFFFFFF))


def workspace_size(cfg: Config, rows: int, cols: int) -> int:
    c = cfg.c()
    return int(_lib.load().fp4q_workspace_size(ctypes.byref(c), rows, cols))


def alloc_workspace(cfg: Config, rows: int, cols: int, device=None):
    torch = _torch()
    n = workspace_size(cfg, rows, cols)
    if n == 0:
        return None
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


@dataclass
class Quantized:
    codes: object          # uint8 [rows, cols/2]
    scales: object         # float32 or uint8
    tensor_scale: object   # float32 [1] (E4M3 scales) or None
    dequant: object        # bf16 [rows, cols] or None
    workspace: object      # uint8 workspace (holds statistics) or None


def _alloc_outputs(cfg: Config, rows, cols, device):
    torch = _torch()
    codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=device)
    if cfg.scale == FP4Q_SCALE_FP32_1x16:
        scales = torch.empty((rows, cols // 16), dtype=torch.float32, device=device)
    else:
        scales = torch.empty((rows, cols // cfg.block), dtype=torch.uint8, device=device)
    return codes, scales


def rht_quantize(cfg: Config, x, *, out: Quantized = None, tensor_scale=None,
                 tensor_scale_given: bool = False, stream=None) -> Quantized:
    """fp4q_rht_quantize. tensor_scale: device float32[1] (E4M3 scales): read when
    tensor_scale_given, else written with the computed alpha."""
    torch = _torch()
    rows, cols, ld = _check_input(x)
    if out is None:
        codes, scales = _alloc_outputs(cfg, rows, cols, x.device)
        deq = torch.empty((rows, cols), dtype=torch.bfloat16, device=x.device) if cfg.dequant else None
        ws = alloc_workspace(cfg, rows, cols, x.device)
        out = Quantized(codes, scales, None, deq, ws)
    if cfg.scale == FP4Q_SCALE_E4M3_1x16_TENSOR:
        if tensor_scale is None:
            tensor_scale = out.tensor_scale if out.tensor_scale is not None else \
                torch.zeros(1, dtype=torch.float32, device=x.device)
        out.tensor_scale = tensor_scale
        _check_buf(out.tensor_scale, "tensor_scale", torch.float32, 1, x.device)
    _check_quantized(cfg, out, rows, cols, x.device, dequant=cfg.dequant)
    c = cfg.c()
    ws = out.workspace
    if ws is not None:
        _check_buf(ws, "workspace", torch.uint8, 0, x.device)
    fn = _lib.load().fp4q_if4_select if cfg.grid == FP4Q_GRID_IF4 else _lib.load().fp4q_rht_quantize
    with torch.cuda.device(x.device):
        st = fn(ctypes.byref(c), _ptr(x), rows, cols, ld, _ptr(out.codes), _ptr(out.scales),
                _ptr(out.tensor_scale), int(bool(tensor_scale_given)), _ptr(out.dequant), _ptr(ws),
                0 if ws is None else ws.numel(), _stream_ptr(stream, x.device))
    _lib.check(st, "fp4q_rht_quantize")
    return out


def rht_quantize_grouped(cfg: Config, x, group_offsets, *, out: Quantized = None,
                         tensor_scales=None, tensor_scales_given: bool = False,
                         stream=None) -> Quantized:
    """fp4q_rht_quantize_grouped. group_offsets: device int64[n_groups + 1] row offsets.
    tensor_scales (E4M3 scales): device float32[n_groups], read when tensor_scales_given, else
    written with each group's computed alpha; returned as Quantized.tensor_scale."""
    torch = _torch()
    rows, cols, ld = _check_input(x)
    _check_buf(group_offsets, "group_offsets", torch.int64, 2, x.device)
    n_groups = int(group_offsets.numel()) - 1
    c = cfg.c()
    if out is None:
        codes, scales = _alloc_outputs(cfg, rows, cols, x.device)
        nws = _lib.load().fp4q_grouped_workspace_size(ctypes.byref(c), n_groups)
        ws = torch.empty(nws, dtype=torch.uint8, device=x.device) if nws else None
        out = Quantized(codes, scales, None, None, ws)
    if tensor_scales is not None:
        out.tensor_scale = tensor_scales
    if cfg.scale == FP4Q_SCALE_E4M3_1x16_TENSOR and out.tensor_scale is None:
        out.tensor_scale = torch.zeros(max(n_groups, 1), dtype=torch.float32, device=x.device)
    if cfg.scale == FP4Q_SCALE_E4M3_1x16_TENSOR:
        _check_buf(out.tensor_scale, "tensor_scales", torch.float32, n_groups, x.device)
    _check_quantized(cfg, out, rows, cols, x.device)
    ws = out.workspace
    if ws is not None:
        _check_buf(ws, "workspace", torch.uint8, 0, x.device)
    with torch.cuda.device(x.device):
        st = _lib.load().fp4q_rht_quantize_grouped(
            ctypes.byref(c), _ptr(x), rows, cols, ld, _ptr(group_offsets), n_groups,
            _ptr(out.codes), _ptr(out.scales), _ptr(out.tensor_scale), int(bool(tensor_scales_given)),
            _ptr(ws), 0 if ws is None else ws.numel(), _stream_ptr(stream, x.device))
    _lib.check(st, "fp4q_rht_quantize_grouped")
    return out


def tensor_scale(cfg: Config, x, *, out=None, workspace=None, stream=None):
    """fp4q_tensor_scale: the FP32 tensor scale alpha of x (E4M3 configurations) -> float32[1]."""
    torch = _torch()
    rows, cols, ld = _check_input(x)
    if out is None:
        out = torch.empty(1, dtype=torch.float32, device=x.device)
    if workspace is None:
        workspace = torch.empty(256, dtype=torch.uint8, device=x.device)
    _check_buf(out, "out", torch.float32, 1, x.device)
    _check_buf(workspace, "workspace", torch.uint8, 0, x.device)
    c = cfg.c()
    with torch.cuda.device(x.device):
        st = _lib.load().fp4q_tensor_scale(ctypes.byref(c), _ptr(x), rows, cols, ld, _ptr(out),
                                           _ptr(workspace), workspace.numel(),
                                           _stream_ptr(stream, x.device))
    _lib.check(st, "fp4q_tensor_scale")
    return out


def if4_select(cfg: Config, x, **kw) -> Quantized:
    """fp4q_if4_select: IF4 with NVFP4 scales (grid/scale in cfg are overridden)."""
    return rht_quantize(replace(cfg, grid=FP4Q_GRID_IF4, scale=FP4Q_SCALE_E4M3_1x16_TENSOR), x, **kw)


@dataclass
class Dual:
    codes_row: object   # uint8 [M, N/2]
    scales_row: object  # float32 [M, N/16]
    codes_col: object   # uint8 [N, M/2]
    scales_col: object  # float32 [N, M/16]


def quantize_dual(row_cfg: Config, col_cfg: Config, dy, *, out: Dual = None, stream=None) -> Dual:
    """fp4q_quantize_dual: dY blocked along N (row) and along M (column) in one pass."""
    torch = _torch()
    M, N, ld = _check_input(dy, "dy")
    if out is None:
        dev = dy.device
        out = Dual(torch.empty((M, N // 2), dtype=torch.uint8, device=dev),
                   torch.empty((M, N // 16), dtype=torch.float32, device=dev),
                   torch.empty((N, M // 2), dtype=torch.uint8, device=dev),
                   torch.empty((N, M // 16), dtype=torch.float32, device=dev))
    for name, dt, n in (("codes_row", torch.uint8, M * (N // 2)), ("scales_row", torch.float32, M * (N // 16)),
                        ("codes_col", torch.uint8, N * (M // 2)), ("scales_col", torch.float32, N * (M // 16))):
        _check_buf(getattr(out, name), name, dt, n, dy.device)
    rc, cc = row_cfg.c(), col_cfg.c()
    with torch.cuda.device(dy.device):
        st = _lib.load().fp4q_quantize_dual(ctypes.byref(rc), ctypes.byref(cc), _ptr(dy), M, N, ld,
                                            _ptr(out.codes_row), _ptr(out.scales_row),
                                            _ptr(out.codes_col), _ptr(out.scales_col), None, 0,
                                            _stream_ptr(stream, dy.device))
    _lib.check(st, "fp4q_quantize_dual")
    return out


def dequantize(cfg: Config, codes, scales, tensor_scale=None, *, inverse_rht: bool = False,
               out=None, stream=None):
    """fp4q_dequantize: codes [rows, cols/2] -> bf16 [rows, cols]."""
    torch = _torch()
    if not (isinstance(codes, torch.Tensor) and codes.dim() == 2):
        raise TypeError("codes must be a 2-D uint8 CUDA tensor [rows, cols/2]")
    rows, cols = codes.shape[0], codes.shape[1] * 2
    dev = codes.device
    _check_buf(codes, "codes", torch.uint8, rows * (cols // 2), dev)
    _check_buf(scales, "scales", _scale_dtype(cfg), rows * (cols // cfg.block), dev)
    if cfg.scale == FP4Q_SCALE_E4M3_1x16_TENSOR:
        _check_buf(tensor_scale, "tensor_scale", torch.float32, 1, dev)
    if out is None:
        out = torch.empty((rows, cols), dtype=torch.bfloat16, device=dev)
    _check_buf(out, "out", torch.bfloat16, rows * cols, dev)
    c = cfg.c()
    with torch.cuda.device(dev):
        st = _lib.load().fp4q_dequantize(ctypes.byref(c), _ptr(codes), _ptr(scales), _ptr(tensor_scale),
                                         rows, cols, int(bool(inverse_rht)), _ptr(out),
                                         _stream_ptr(stream, dev))
    _lib.check(st, "fp4q_dequantize")
    return out


def rht16(x, sign_mask: int, *, out_fp32: bool = False, out=None, stream=None):
    """fp4q_rht16: the rotation alone (bf16 or FP32 output)."""
    torch = _torch()
    rows, cols, ld = _check_input(x)
    if out is None:
        out = torch.empty((rows, cols), dtype=torch.float32 if out_fp32 else torch.bfloat16,
                          device=x.device)
    _check_buf(out, "out", torch.float32 if out_fp32 else torch.bfloat16, rows * cols, x.device)
    with torch.cuda.device(x.device):
        st = _lib.load().fp4q_rht16(_ptr(x), rows, cols, ld, sign_mask, _ptr(out), int(bool(out_fp32)),
                                    _stream_ptr(stream, x.device))
    _lib.check(st, "fp4q_rht16")
    return out


def device_status(clear: bool = False, stream=None) -> int:
    """fp4q_device_status: the library's sticky device status bits (0 when all is well)."""
    v = ctypes.c_int32(0)
    _lib.check(_lib.load().fp4q_device_status(ctypes.byref(v), int(bool(clear)), _stream_ptr(stream)),
               "fp4q_device_status")
    return int(v.value)


def stats(workspace, stream=None) -> dict:
    """fp4q_stats: reduce and fetch the statistics a stats-enabled call left in `workspace`."""
    torch = _torch()
    _check_buf(workspace, "workspace", torch.uint8, 0, getattr(workspace, "device", None))
    res = _lib.fp4q_stats_t()
    with torch.cuda.device(workspace.device):
        st = _lib.load().fp4q_stats(_ptr(workspace), workspace.numel(), ctypes.byref(res),
                                    _stream_ptr(stream, workspace.device))
    _lib.check(st, "fp4q_stats")
    out = {}
    for name, _ in _lib.fp4q_stats_t._fields_:
        v = getattr(res, name)
        out[name] = list(v) if hasattr(v, "__len__") else v
    return out


def gemm_nvfp4(a: Quantized, b: Quantized, *, out=None, stream=None):
    """fp4q_gemm_nvfp4: out[m, n] = alpha_a alpha_b sum_k A[m, k] B[n, k] in bf16, from two NVFP4
    quantizations (E2M1 codes, E4M3 scales in the MMA layout, tensor scales) used unchanged."""
    torch = _torch()
    for name, q in (("a", a), ("b", b)):
        if not isinstance(q, Quantized) or q.tensor_scale is None:
            raise TypeError("%s must be the Quantized result of an NVFP4 quantization" % name)
    M, K2 = a.codes.shape
    N = b.codes.shape[0]
    K = 2 * K2
    dev = a.codes.device
    _check_buf(a.codes, "a.codes", torch.uint8, M * K2, dev)
    _check_buf(b.codes, "b.codes", torch.uint8, N * K2, dev)
    _check_buf(a.scales, "a.scales", torch.uint8, M * (K // 16), dev)
    _check_buf(b.scales, "b.scales", torch.uint8, N * (K // 16), dev)
    _check_buf(a.tensor_scale, "a.tensor_scale", torch.float32, 1, dev)
    _check_buf(b.tensor_scale, "b.tensor_scale", torch.float32, 1, dev)
    if b.codes.shape[1] != K2:
        raise ValueError("a and b must have the same K")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    if not (isinstance(out, torch.Tensor) and out.is_cuda and out.dtype == torch.bfloat16 and out.dim() == 2
            and out.stride(1) == 1 and out.shape[0] == M and out.shape[1] == N):
        raise TypeError("out must be a bf16 CUDA tensor [M, N] with unit column stride")
    if out.device != dev:
        raise ValueError("out is on %s but the operands are on %s" % (out.device, dev))
    ldo = out.stride(0) if M > 1 else N
    with torch.cuda.device(dev):
        st = _lib.load().fp4q_gemm_nvfp4(_ptr(a.codes), _ptr(a.scales), _ptr(a.tensor_scale), _ptr(b.codes),
                                         _ptr(b.scales), _ptr(b.tensor_scale), M, N, K, _ptr(out), ldo,
                                         _stream_ptr(stream, dev))
    _lib.check(st, "fp4q_gemm_nvfp4")
    return out



def gemm_mxfp4(a: Quantized, b: Quantized, *, out=None, stream=None):
    """fp4q_gemm_mxfp4: out[m, n] = sum_k A[m, k] B[n, k] in bf16, from two MXFP4 quantizations
    (E2M1 codes, UE8M0 scales in the MMA layout) used unchanged."""
    torch = _torch()
    for name, q in (("a", a), ("b", b)):
        if not isinstance(q, Quantized):
            raise TypeError("%s must be the Quantized result of an MXFP4 quantization" % name)
    M, K2 = a.codes.shape
    N = b.codes.shape[0]
    K = 2 * K2
    dev = a.codes.device
    _check_buf(a.codes, "a.codes", torch.uint8, M * K2, dev)
    _check_buf(b.codes, "b.codes", torch.uint8, N * K2, dev)
    _check_buf(a.scales, "a.scales", torch.uint8, M * (K // 32), dev)
    _check_buf(b.scales, "b.scales", torch.uint8, N * (K // 32), dev)
    if b.codes.shape[1] != K2:
        raise ValueError("a and b must have the same K")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    if not (isinstance(out, torch.Tensor) and out.is_cuda and out.dtype == torch.bfloat16 and out.dim() == 2
            and out.stride(1) == 1 and out.shape[0] == M and out.shape[1] == N):
        raise TypeError("out must be a bf16 CUDA tensor [M, N] with unit column stride")
    if out.device != dev:
        raise ValueError("out is on %s but the operands are on %s" % (out.device, dev))
    ldo = out.stride(0) if M > 1 else N
    with torch.cuda.device(dev):
        st = _lib.load().fp4q_gemm_mxfp4(_ptr(a.codes), _ptr(a.scales), _ptr(b.codes), _ptr(b.scales), M, N, K,
                                         _ptr(out), ldo, _stream_ptr(stream, dev))
    _lib.check(st, "fp4q_gemm_mxfp4")
    return out