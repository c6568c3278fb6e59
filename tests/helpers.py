"""Shared test helpers: mapping the library's config onto the oracle's, host<->device copies."""
import numpy as np

import oracle as O
import block_scaled_bit_rht16_b200 as fq

GRID = {fq.FP4Q_GRID_E2M1: O.GRID_E2M1, fq.FP4Q_GRID_E1M2: O.GRID_E1M2,
        fq.FP4Q_GRID_INT4: O.GRID_INT4, fq.FP4Q_GRID_IF4: O.GRID_IF4}
SCALE = {fq.FP4Q_SCALE_FP32_1x16: O.SCALE_FP32_1x16, fq.FP4Q_SCALE_E4M3_1x16_TENSOR: O.SCALE_E4M3_1x16,
         fq.FP4Q_SCALE_UE8M0_1x32: O.SCALE_UE8M0_1x32}
ROUND = {fq.FP4Q_ROUND_RTNE: O.ROUND_RTNE, fq.FP4Q_ROUND_SR: O.ROUND_SR}


RESTRICTED = {4: O.GRID_E2M1_MAX4, 3: O.GRID_E2M1_MAX3, 2: O.GRID_E2M1_MAX2}


def ocfg(cfg: "fq.Config") -> O.OracleConfig:
    grid = RESTRICTED[cfg.e2m1_max] if cfg.e2m1_max else GRID[cfg.grid]
    return O.OracleConfig(grid=grid, scale=SCALE[cfg.scale], round=ROUND[cfg.round],
                          rht=cfg.rht, sign_mask=cfg.sign_mask, sr_stream=cfg.sr_stream,
                          sr_seed=cfg.sr_seed)


def to_dev(bits: np.ndarray, ld: int = None):
    """uint16 bf16 bit patterns -> CUDA bf16 tensor (optionally with a wider row pitch)."""
    import torch
    bits = np.ascontiguousarray(bits)
    t = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)
    if ld is not None and ld != bits.shape[1]:
        big = torch.zeros((bits.shape[0], ld), dtype=torch.bfloat16)
        big[:, :bits.shape[1]] = t
        return big.cuda()[:, :bits.shape[1]]
    return t.cuda()


def bf16_bits(t) -> np.ndarray:
    import torch
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def host(t) -> np.ndarray:
    return t.detach().cpu().numpy()
