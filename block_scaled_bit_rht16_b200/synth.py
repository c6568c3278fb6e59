"""Seeded synthetic inputs shaped like the linear-layer tensors the UFP4 / IF4 pages discuss.

This module only draws random numbers and rounds them to bfloat16; it holds none of the
quantizer's arithmetic. Both the CUDA path's tests/benchmark and the CPU oracle's tests take
their inputs from here, so the two see identical bytes.

Recipe: numpy ``default_rng(seed)`` (PCG64) draws FP32 values, which are rounded to bfloat16
(round to nearest even on the bit pattern) and returned as uint16 bit patterns.
Every input has a seed tag t (below): data seed 1000 + t, rotation sign seed 0x5EED0000 + t;
the stochastic-rounding seed is 0x5A5A0003.

Inputs (tag; the standard deviations are the second parameter of N(., .)):
  outlier_activation      1  activation [512, 2048], N(0,1), 8 distinct columns x50
  dense_linear_operands   2  dense-1.5B-like operands: X [8192, 2048] Student-t nu=4;
                             W [8192, 2048] N(0, 0.02)
  backward_dy             3  dY [8192, 8192] N(0, 1e-3), 0.01% of entries (distinct positions) x100
  laplace_format_tensor   4  [16384, 5120] Laplace(0, 1)
  moe_expert              5  MoE experts [64, 2048, 7168], expert e ~ N(0, sigma_e),
                             sigma_e = 10^U(-1, 1) (moe_expert_sigmas)
  dense_layer_rows        5  dense [32768, 8192] N(0, 1)
"""
import numpy as np

SR_SEED = 0x5A5A0003


def data_seed(tag: int) -> int:
    return 1000 + tag


def sign_seed(tag: int) -> int:
    return 0x5EED0000 + tag


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """FP32 -> bfloat16 bit patterns, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    return ((u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def outlier_activation(seed: int = data_seed(1), rows: int = 512, cols: int = 2048) -> np.ndarray:
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, cols), dtype=np.float32)
    cols_out = rng.choice(cols, size=8, replace=False)
    x[:, cols_out] *= np.float32(50.0)
    return to_bf16_bits(x)


def dense_linear_operands(seed: int = data_seed(2), rows: int = 8192, cols: int = 2048):
    """Returns (X, W): X Student-t(4), W N(0, 0.02)."""
    rng = np.random.default_rng(seed)
    x = rng.standard_t(4.0, size=(rows, cols)).astype(np.float32)
    w = rng.normal(0.0, 0.02, size=(rows, cols)).astype(np.float32)
    return to_bf16_bits(x), to_bf16_bits(w)


def backward_dy(seed: int = data_seed(3), rows: int = 8192, cols: int = 8192,
              outlier_fraction: float = 1e-4) -> np.ndarray:
    rng = np.random.default_rng(seed)
    x = rng.normal(0.0, 1e-3, size=(rows, cols)).astype(np.float32)
    n_out = int(round(outlier_fraction * rows * cols))
    pos = rng.choice(rows * cols, size=n_out, replace=False)
    x.reshape(-1)[pos] *= np.float32(100.0)
    return to_bf16_bits(x)


def laplace_format_tensor(seed: int = data_seed(4), rows: int = 16384, cols: int = 5120) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return to_bf16_bits(rng.laplace(0.0, 1.0, size=(rows, cols)).astype(np.float32))


def moe_expert_sigmas(seed: int = data_seed(5), experts: int = 64) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return (10.0 ** rng.uniform(-1.0, 1.0, size=experts)).astype(np.float32)


def moe_expert(e: int, seed: int = data_seed(5), tokens: int = 2048, hidden: int = 7168,
                     experts: int = 64) -> np.ndarray:
    """One expert's [tokens, hidden] slab (independent stream per expert)."""
    sigma = moe_expert_sigmas(seed, experts)[e]
    rng = np.random.default_rng([seed, 1, e])
    return to_bf16_bits(rng.standard_normal((tokens, hidden), dtype=np.float32) * sigma)


def dense_layer_rows(r0: int, r1: int, seed: int = data_seed(5), cols: int = 8192,
                         chunk: int = 1024) -> np.ndarray:
    """Rows [r0, r1) of the dense [32768, 8192] N(0,1) tensor, drawn in fixed 1024-row chunks
    so any row range is reproducible on its own."""
    out = np.empty((r1 - r0, cols), dtype=np.uint16)
    c0 = (r0 // chunk) * chunk
    while c0 < r1:
        rng = np.random.default_rng([seed, 2, c0 // chunk])
        blk = to_bf16_bits(rng.standard_normal((chunk, cols), dtype=np.float32))
        a, b = max(r0, c0), min(r1, c0 + chunk)
        out[a - r0:b - r0] = blk[a - c0:b - c0]
        c0 += chunk
    return out


def small(seed: int, rows: int, cols: int, kind: str = "normal", scale: float = 1.0) -> np.ndarray:
    """Small seeded matrices for parity cases: kind in normal | t4 | laplace | uniform."""
    rng = np.random.default_rng(seed)
    if kind == "normal":
        x = rng.standard_normal((rows, cols), dtype=np.float32)
    elif kind == "t4":
        x = rng.standard_t(4.0, size=(rows, cols)).astype(np.float32)
    elif kind == "laplace":
        x = rng.laplace(0.0, 1.0, size=(rows, cols)).astype(np.float32)
    elif kind == "uniform":
        x = rng.uniform(-1.0, 1.0, size=(rows, cols)).astype(np.float32)
    else:
        raise ValueError(kind)
    return to_bf16_bits(x * np.float32(scale))
