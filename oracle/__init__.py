"""CPU oracle for the fused RHT16 + block-scaled 4-bit quantizer -- TEST INFRASTRUCTURE.

The arithmetic lives in ``fp4q_oracle.c`` (plain C, one IEEE binary32 operation per source
operation, no FMA contraction); this module only marshals numpy arrays into it and computes
the derived statistics with the plain formulas. Only the test suite, the package smoke check
and the benchmark's CPU-baseline leg may import it; the product path never does.

Configuration constants here are the oracle's own; callers map the library's config onto them.
"""
import ctypes
import math
from dataclasses import dataclass

import numpy as np

from . import build as _build

GRID_E2M1, GRID_E1M2, GRID_INT4, GRID_IF4 = 0, 1, 2, 3
GRID_E2M1_MAX4, GRID_E2M1_MAX3, GRID_E2M1_MAX2 = 4, 5, 6   # range-restricted E2M1
SCALE_FP32_1x16, SCALE_E4M3_1x16, SCALE_UE8M0_1x32 = 0, 1, 2
ROUND_RTNE, ROUND_SR = 0, 1

ST_SUM_Y2, ST_SUM_ERR2, ST_SUM_YXHAT, ST_N = 0, 1, 2, 3
ST_CELL_N, ST_CELL_ERR, ST_IF4_FP4, ST_BLOCKS, ST_LEN = 4, 12, 20, 21, 24


class _Cfg(ctypes.Structure):
    _fields_ = [("grid", ctypes.c_int32), ("scale", ctypes.c_int32), ("round", ctypes.c_int32),
                ("rht", ctypes.c_int32), ("sign_mask", ctypes.c_uint32),
                ("sr_stream", ctypes.c_uint32), ("sr_seed", ctypes.c_uint64)]


@dataclass(frozen=True)
class OracleConfig:
    grid: int = GRID_E1M2
    scale: int = SCALE_FP32_1x16
    round: int = ROUND_RTNE
    rht: int = 1
    sign_mask: int = 0
    sr_stream: int = 0
    sr_seed: int = 0

    def _c(self):
        return _Cfg(self.grid, self.scale, self.round, self.rht, self.sign_mask & 0xFFFFFFFF,
                    self.sr_stream & 0xFFFFFFFF, self.sr_seed & 0xFFFFFFFFFFFFFFFF)


_lib = ctypes.CDLL(_build.build())
_P = ctypes.c_void_p
_I64 = ctypes.c_int64
for name, res, args in [
    ("orc_splitmix64", ctypes.c_uint64, [ctypes.c_uint64]),
    ("orc_sr_bits", ctypes.c_uint32, [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint64]),
    ("orc_sign_mask_from_seed", ctypes.c_uint32, [ctypes.c_uint64]),
    ("orc_grid_magnitudes", ctypes.c_int, [ctypes.c_int, _P]),
    ("orc_decode_nibble", ctypes.c_double, [ctypes.c_int, ctypes.c_uint8]),
    ("orc_round_rtne", ctypes.c_uint8, [ctypes.c_int, ctypes.c_float]),
    ("orc_round_sr", ctypes.c_uint8, [ctypes.c_int, ctypes.c_float, ctypes.c_uint32]),
    ("orc_round_rtne_n", None, [ctypes.c_int, _P, _I64, _P]),
    ("orc_round_sr_n", None, [ctypes.c_int, _P, _P, _I64, _P]),
    ("orc_e4m3_encode", ctypes.c_uint8, [ctypes.c_float]),
    ("orc_e4m3_encode_n", None, [_P, _I64, _P]),
    ("orc_e4m3_decode", ctypes.c_float, [ctypes.c_uint8]),
    ("orc_mx_exponent", ctypes.c_int, [ctypes.c_float]),
    ("orc_f32_to_bf16_n", None, [_P, _I64, _P]),
    ("orc_sylvester_h16", None, [_P]),
    ("orc_rht16", None, [_P, ctypes.c_uint32, _P]),
    ("orc_inverse_rht16", None, [_P, ctypes.c_uint32, _P]),
    ("orc_tensor_amax", ctypes.c_float, [ctypes.POINTER(_Cfg), _P, _I64, _I64, _I64]),
    ("orc_quantize", ctypes.c_int, [ctypes.POINTER(_Cfg), _P, _I64, _I64, _I64, _I64, _P, _P,
                                    _P, ctypes.c_int32, _P, _P]),
    ("orc_dequantize", ctypes.c_int, [ctypes.POINTER(_Cfg), _P, _P, ctypes.c_float, _I64, _I64,
                                      ctypes.c_int32, _P]),
    ("orc_rht16_rows", ctypes.c_int, [_P, _I64, _I64, _I64, ctypes.c_uint32, _P, _P]),
]:
    fn = getattr(_lib, name)
    fn.restype = res
    fn.argtypes = args


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


# ---------------------------------------------------------------- scalar rules

def splitmix64(x: int) -> int:
    return int(_lib.orc_splitmix64(x & 0xFFFFFFFFFFFFFFFF))


def sr_bits(seed: int, stream: int, idx: int) -> int:
    return int(_lib.orc_sr_bits(seed & 0xFFFFFFFFFFFFFFFF, stream, idx))


def sign_mask_from_seed(seed: int) -> int:
    return int(_lib.orc_sign_mask_from_seed(seed & 0xFFFFFFFFFFFFFFFF))


def grid_magnitudes(grid: int) -> np.ndarray:
    """The magnitudes a grid rounds to, by magnitude code (8; 7, 6, 5 for restricted E2M1)."""
    g = np.zeros(8, dtype=np.float64)
    n = _lib.orc_grid_magnitudes(grid, _ptr(g))
    assert n > 0
    return g[:n]


def decode_nibble(grid: int, nib: int) -> float:
    return float(_lib.orc_decode_nibble(grid, nib))


def round_rtne(grid: int, v) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, dtype=np.uint8)
    _lib.orc_round_rtne_n(grid, _ptr(v), v.size, _ptr(out))
    return out


def round_sr(grid: int, v, u) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32)
    u = np.ascontiguousarray(u, dtype=np.uint32)
    assert v.shape == u.shape
    out = np.empty(v.shape, dtype=np.uint8)
    _lib.orc_round_sr_n(grid, _ptr(v), _ptr(u), v.size, _ptr(out))
    return out


def e4m3_encode(x) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint8)
    _lib.orc_e4m3_encode_n(_ptr(x), x.size, _ptr(out))
    return out


def e4m3_decode(b: int) -> float:
    return float(_lib.orc_e4m3_decode(b))


def mx_exponent(amax: float) -> int:
    return int(_lib.orc_mx_exponent(amax))


def f32_to_bf16(x) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint16)
    _lib.orc_f32_to_bf16_n(_ptr(x), x.size, _ptr(out))
    return out


def sylvester_h16() -> np.ndarray:
    h = np.zeros((16, 16), dtype=np.int32)
    _lib.orc_sylvester_h16(_ptr(h))
    return h


def rht16(x, mask: int) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    assert x.shape == (16,)
    y = np.empty(16, dtype=np.float32)
    _lib.orc_rht16(_ptr(x), mask, _ptr(y))
    return y


def inverse_rht16(y, mask: int) -> np.ndarray:
    y = np.ascontiguousarray(y, dtype=np.float32)
    assert y.shape == (16,)
    x = np.empty(16, dtype=np.float32)
    _lib.orc_inverse_rht16(_ptr(y), mask, _ptr(x))
    return x


# ---------------------------------------------------------------- tensor-level quantizer

def block_size(cfg: OracleConfig) -> int:
    return 32 if cfg.scale == SCALE_UE8M0_1x32 else 16


def tensor_amax(cfg: OracleConfig, x: np.ndarray) -> float:
    assert x.dtype == np.uint16 and x.ndim == 2 and x.strides[1] == 2
    c = cfg._c()
    return float(_lib.orc_tensor_amax(ctypes.byref(c), _ptr(x), x.shape[0], x.shape[1],
                                      x.strides[0] // 2))


def quantize(cfg: OracleConfig, x: np.ndarray, *, row0: int = 0, tensor_scale=None,
             dequant: bool = False, stats: bool = False) -> dict:
    """Quantize a bfloat16 matrix (given as uint16 bits, [rows, cols], unit column stride).

    Returns dict(codes [rows, cols/2] u8, scales (f32 or u8), tensor_scale (float or None),
    dequant (uint16 bf16 bits or None), stats_raw (float64[ST_LEN] or None)).
    ``tensor_scale`` (E4M3 scales only): alpha to use; None computes it from this matrix.
    """
    assert x.dtype == np.uint16 and x.ndim == 2 and x.strides[1] == 2
    rows, cols = x.shape
    bs = block_size(cfg)
    codes = np.zeros((rows, cols // 2), dtype=np.uint8)
    if cfg.scale == SCALE_FP32_1x16:
        scales = np.zeros((rows, cols // bs), dtype=np.float32)
    else:
        scales = np.zeros((rows, cols // bs), dtype=np.uint8)
    ts = np.zeros(1, dtype=np.float32)
    given = 0
    if tensor_scale is not None:
        ts[0] = tensor_scale
        given = 1
    deq = np.zeros((rows, cols), dtype=np.uint16) if dequant else None
    st = np.zeros(ST_LEN, dtype=np.float64) if stats else None
    c = cfg._c()
    rc = _lib.orc_quantize(ctypes.byref(c), _ptr(x), rows, cols, x.strides[0] // 2, row0,
                           _ptr(codes), _ptr(scales), _ptr(ts), given, _ptr(deq), _ptr(st))
    if rc != 0:
        raise ValueError("oracle rejected the configuration or shape")
    return dict(codes=codes, scales=scales,
                tensor_scale=float(ts[0]) if cfg.scale == SCALE_E4M3_1x16 else None,
                dequant=deq, stats_raw=st)


def dequantize(cfg: OracleConfig, codes: np.ndarray, scales: np.ndarray, tensor_scale: float,
               rows: int, cols: int, inverse_rht: bool = False) -> np.ndarray:
    codes = np.ascontiguousarray(codes)
    scales = np.ascontiguousarray(scales)
    out = np.zeros((rows, cols), dtype=np.uint16)
    c = cfg._c()
    rc = _lib.orc_dequantize(ctypes.byref(c), _ptr(codes), _ptr(scales),
                             float(tensor_scale or 0.0), rows, cols, int(inverse_rht), _ptr(out))
    if rc != 0:
        raise ValueError("oracle rejected the configuration or shape")
    return out


def rht16_rows(x: np.ndarray, mask: int):
    """The rotation alone: returns (FP32 [rows, cols], bf16 bits [rows, cols])."""
    assert x.dtype == np.uint16 and x.ndim == 2 and x.strides[1] == 2
    rows, cols = x.shape
    yf = np.zeros((rows, cols), dtype=np.float32)
    yb = np.zeros((rows, cols), dtype=np.uint16)
    rc = _lib.orc_rht16_rows(_ptr(x), rows, cols, x.strides[0] // 2, mask, _ptr(yf), _ptr(yb))
    if rc != 0:
        raise ValueError("oracle rejected the shape")
    return yf, yb


def finalize_stats(raw: np.ndarray) -> dict:
    """Derived statistics from a raw record (R15): SQNR in dB [UFP4-A, RHT section],
    signal attenuation alpha = <xhat, y>/|y|^2 [UFP4-A, compounding section], MSE, per-cell
    mean signed error in scaled units [UFP4-A, E2M1 section], IF4 FP4 fraction [IF4 6.2]."""
    y2, e2, yx, n = raw[ST_SUM_Y2], raw[ST_SUM_ERR2], raw[ST_SUM_YXHAT], raw[ST_N]
    cell_n = raw[ST_CELL_N:ST_CELL_N + 8]
    cell_e = raw[ST_CELL_ERR:ST_CELL_ERR + 8]
    sqnr = math.inf if e2 == 0 else (10.0 * math.log10(y2 / e2) if y2 > 0 else -math.inf)
    with np.errstate(invalid="ignore", divide="ignore"):
        cell_mean = np.where(cell_n > 0, cell_e / np.maximum(cell_n, 1), np.nan)
    blocks = raw[ST_BLOCKS]
    return dict(sqnr_db=sqnr, alpha=(yx / y2 if y2 > 0 else 1.0), mse=(e2 / n if n else 0.0),
                nmse=(e2 / y2 if y2 > 0 else 0.0), n=n, cell_count=cell_n.copy(),
                cell_mean_err=cell_mean, if4_fp4_fraction=(raw[ST_IF4_FP4] / blocks if blocks else 0.0),
                blocks=blocks)
