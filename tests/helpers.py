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


class Canaries:
    """Output buffers placed between two guard bands of a known byte pattern (PAD bytes each), so
    that a kernel writing past either end of an output changes a band. check() asserts every band
    is intact. The bands keep 256-byte alignment, so outputs stay as aligned as torch's own."""
    PAD = 256
    FILL = 0xA7

    def __init__(self, device="cuda"):
        self.device = device
        self.raws = []

    def empty(self, shape, dtype):
        import torch
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        raw = torch.full((n + 2 * self.PAD,), self.FILL, dtype=torch.uint8, device=self.device)
        self.raws.append((raw, n))
        return raw[self.PAD:self.PAD + n].view(dtype).view(shape)

    def check(self):
        import torch
        torch.cuda.synchronize()
        for i, (raw, n) in enumerate(self.raws):
            lo = raw[:self.PAD].cpu().numpy()
            hi = raw[self.PAD + n:].cpu().numpy()
            bad_lo = np.nonzero(lo != self.FILL)[0]
            bad_hi = np.nonzero(hi != self.FILL)[0]
            assert bad_lo.size == 0, "buffer %d (%d bytes): %d bytes written before its start" % (i, n, bad_lo.size)
            assert bad_hi.size == 0, "buffer %d (%d bytes): %d bytes written past its end (first at +%d)" % (
                i, n, bad_hi.size, int(bad_hi[0]) if bad_hi.size else -1)


def guarded_quantized(cfg, rows, cols, guard):
    """fq.Quantized outputs of a row quantizer (codes, scales, tensor scale, dequant,
    workspace), each between guard bands."""
    import torch
    codes = guard.empty((rows, cols // 2), torch.uint8)
    sdt = torch.float32 if cfg.scale == fq.FP4Q_SCALE_FP32_1x16 else torch.uint8
    scales = guard.empty((rows, cols // cfg.block), sdt)
    deq = guard.empty((rows, cols), torch.bfloat16) if cfg.dequant else None
    nws = fq.workspace_size(cfg, rows, cols)
    ws = guard.empty((nws,), torch.uint8) if nws else None
    ts = guard.empty((1,), torch.float32) if cfg.scale == fq.FP4Q_SCALE_E4M3_1x16_TENSOR else None
    return fq.Quantized(codes, scales, ts, deq, ws)


def guarded_dual(M, N, guard):
    import torch
    return fq.Dual(guard.empty((M, N // 2), torch.uint8), guard.empty((M, N // 16), torch.float32),
                   guard.empty((N, M // 2), torch.uint8), guard.empty((N, M // 16), torch.float32))


def oracle_rows(oc, bits, tensor_scale=None, dequant=False, stats=False, chunk=256, threads=None):
    """The oracle over every row of `bits`, in row chunks (row0 set, so stochastic rounding
    draws its global indices) run on a thread pool (the ctypes calls release the GIL).
    Returns codes, scales and, when asked, dequant and the summed raw statistics."""
    import concurrent.futures as cf
    import os
    M = bits.shape[0]
    starts = list(range(0, M, chunk))

    def one(r0):
        return O.quantize(oc, np.ascontiguousarray(bits[r0:r0 + chunk]), row0=r0,
                          tensor_scale=tensor_scale, dequant=dequant, stats=stats)
    threads = threads or len(os.sched_getaffinity(0))
    with cf.ThreadPoolExecutor(max_workers=threads) as ex:
        parts = list(ex.map(one, starts))
    out = {"codes": np.concatenate([p["codes"] for p in parts]),
           "scales": np.concatenate([p["scales"] for p in parts])}
    if dequant:
        out["dequant"] = np.concatenate([p["dequant"] for p in parts])
    if stats:
        out["stats_raw"] = np.sum([p["stats_raw"] for p in parts], axis=0)
    return out
