"""ctypes view of libfp4q.so: the structs and entry points of include/fp4q.h, unchanged.

Loading fails loudly (ImportError) when the library has not been built: there is no fallback.
"""
import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libfp4q.so")

FP4Q_OK, FP4Q_ERR_INVALID_ARG, FP4Q_ERR_SHAPE, FP4Q_ERR_ALIGN = 0, 1, 2, 3
FP4Q_ERR_UNSUPPORTED, FP4Q_ERR_WORKSPACE, FP4Q_ERR_CUDA, FP4Q_ERR_TIMEOUT = 4, 5, 6, 7
FP4Q_GRID_E2M1, FP4Q_GRID_E1M2, FP4Q_GRID_INT4, FP4Q_GRID_IF4 = 0, 1, 2, 3
FP4Q_SCALE_FP32_1x16, FP4Q_SCALE_E4M3_1x16_TENSOR, FP4Q_SCALE_UE8M0_1x32 = 0, 1, 2
FP4Q_ROUND_RTNE, FP4Q_ROUND_SR = 0, 1
FP4Q_OUT_CODES, FP4Q_OUT_DEQUANT, FP4Q_OUT_STATS, FP4Q_OUT_SCALES_MMA = 1, 2, 4, 8

# Every function include/fp4q.h declares (checked by the host tests against the header).
EXPORTS = ["fp4q_status_string", "fp4q_sign_mask_from_seed", "fp4q_workspace_size",
           "fp4q_rht_quantize", "fp4q_quantize_dual", "fp4q_dequantize", "fp4q_if4_select",
           "fp4q_stats", "fp4q_rht16", "fp4q_check_division", "fp4q_device_status",
           "fp4q_check_wait_timeout", "fp4q_tensor_scale", "fp4q_rht_quantize_noalloc",
           "fp4q_grouped_workspace_size", "fp4q_rht_quantize_grouped", "fp4q_check_conversions",
           "fp4q_gemm_nvfp4", "fp4q_gemm_mxfp4"]


class fp4q_config(ctypes.Structure):
    _fields_ = [("grid", ctypes.c_int32), ("scale", ctypes.c_int32), ("round", ctypes.c_int32),
                ("rht", ctypes.c_int32), ("sign_mask", ctypes.c_uint32),
                ("sr_stream", ctypes.c_uint32), ("sr_seed", ctypes.c_uint64),
                ("outputs", ctypes.c_uint32), ("e2m1_max", ctypes.c_uint32)]


class fp4q_stats_t(ctypes.Structure):
    _fields_ = [("sum_y2", ctypes.c_double), ("sum_err2", ctypes.c_double),
                ("sum_y_xhat", ctypes.c_double), ("n", ctypes.c_double),
                ("cell_count", ctypes.c_double * 8), ("cell_err", ctypes.c_double * 8),
                ("if4_fp4_blocks", ctypes.c_double), ("blocks", ctypes.c_double),
                ("sqnr_db", ctypes.c_double), ("alpha", ctypes.c_double),
                ("mse", ctypes.c_double), ("nmse", ctypes.c_double),
                ("cell_mean_err", ctypes.c_double * 8), ("if4_fp4_fraction", ctypes.c_double),
                ("status", ctypes.c_int32), ("reserved", ctypes.c_int32)]


_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_CFG = ctypes.POINTER(fp4q_config)
SIGNATURES = {
    "fp4q_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "fp4q_sign_mask_from_seed": (ctypes.c_uint32, [ctypes.c_uint64]),
    "fp4q_workspace_size": (ctypes.c_size_t, [_CFG, _I64, _I64]),
    "fp4q_rht_quantize": (ctypes.c_int, [_CFG, _P, _I64, _I64, _I64, _P, _P, _P, ctypes.c_int32,
                                         _P, _P, ctypes.c_size_t, _P]),
    "fp4q_quantize_dual": (ctypes.c_int, [_CFG, _CFG, _P, _I64, _I64, _I64, _P, _P, _P, _P, _P,
                                          ctypes.c_size_t, _P]),
    "fp4q_dequantize": (ctypes.c_int, [_CFG, _P, _P, _P, _I64, _I64, ctypes.c_int32, _P, _P]),
    "fp4q_if4_select": (ctypes.c_int, [_CFG, _P, _I64, _I64, _I64, _P, _P, _P, ctypes.c_int32,
                                       _P, _P, ctypes.c_size_t, _P]),
    "fp4q_stats": (ctypes.c_int, [_P, ctypes.c_size_t, ctypes.POINTER(fp4q_stats_t), _P]),
    "fp4q_rht16": (ctypes.c_int, [_P, _I64, _I64, _I64, ctypes.c_uint32, _P, ctypes.c_int32, _P]),
    "fp4q_check_division": (ctypes.c_int, [ctypes.c_uint64, ctypes.c_uint64, _P, _P]),
    "fp4q_check_conversions": (ctypes.c_int, [_P, _P]),
    "fp4q_gemm_nvfp4": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _P, _I64, _P]),
    "fp4q_gemm_mxfp4": (ctypes.c_int, [_P, _P, _P, _P, _I64, _I64, _I64, _P, _I64, _P]),
    "fp4q_device_status": (ctypes.c_int, [ctypes.POINTER(ctypes.c_int32), ctypes.c_int32, _P]),
    "fp4q_check_wait_timeout": (ctypes.c_int, [ctypes.c_uint64, _P]),
    "fp4q_tensor_scale": (ctypes.c_int, [_CFG, _P, _I64, _I64, _I64, _P, _P, ctypes.c_size_t, _P]),
    "fp4q_rht_quantize_noalloc": (ctypes.c_int, [_CFG, _P, _I64, _I64, _I64, _P, _P, _P,
                                                 ctypes.c_int32, _P, _P]),
    "fp4q_grouped_workspace_size": (ctypes.c_size_t, [_CFG, ctypes.c_int32]),
    "fp4q_rht_quantize_grouped": (ctypes.c_int, [_CFG, _P, _I64, _I64, _I64, _P, ctypes.c_int32,
                                                 _P, _P, _P, ctypes.c_int32, _P, ctypes.c_size_t,
                                                 _P]),
}

_lib = None


def load():
    """The loaded library (cached). Raises ImportError if libfp4q.so is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError("libfp4q.so is not built (python -m block_scaled_bit_rht16_b200.build)")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


class Fp4qError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = load().fp4q_status_string(status).decode()
        super().__init__("%s: %s (status %d)" % (where, msg, status))
        self.status = status


def check(status: int, where: str) -> None:
    if status != FP4Q_OK:
        raise Fp4qError(status, where)
