"""Prints the oracle's statistics on the full-size synthetic inputs, for comparison with the
values the pages print without their data (UFP4 explainer, RHT section: SQNR across the
rotation; IF4 page, section 2.2 table: format MSEs; section 6.2: IF4 FP4-block share).
Bit-exact parity makes these the library's values too. Run: python tests/format_stats_report.py
(about a minute on 8 cores). Not collected by pytest."""
import concurrent.futures as cf
import json
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import oracle as O  # noqa: E402
from block_scaled_bit_rht16_b200 import synth  # noqa: E402


def _chunks(n, c=512):
    return [(r, min(r + c, n)) for r in range(0, n, c)]


def _stats(cfg, x, tensor_scale=None):
    def one(rr):
        r0, r1 = rr
        return O.quantize(cfg, np.ascontiguousarray(x[r0:r1]), row0=r0, tensor_scale=tensor_scale,
                          stats=True)["stats_raw"]
    with cf.ThreadPoolExecutor(os.cpu_count()) as ex:
        return O.finalize_stats(sum(ex.map(one, _chunks(x.shape[0]))))


def _tensor_amax(cfg, x):
    def one(rr):
        return O.tensor_amax(cfg, np.ascontiguousarray(x[rr[0]:rr[1]]))
    with cf.ThreadPoolExecutor(os.cpu_count()) as ex:
        return max(ex.map(one, _chunks(x.shape[0])))


def main():
    out = {}
    x = synth.outlier_activation()
    mask = O.sign_mask_from_seed(synth.sign_seed(1))
    for name, grid in (("E2M1", O.GRID_E2M1), ("E1M2", O.GRID_E1M2)):
        for rht in (0, 1):
            st = _stats(O.OracleConfig(grid=grid, rht=rht, sign_mask=mask if rht else 0), x)
            out["outlier_activation %s %s" % (name, "RHT16" if rht else "no rotation")] = {
                "sqnr_db": round(st["sqnr_db"], 2), "alpha": round(st["alpha"], 5),
                "cell_mean_err": [None if np.isnan(v) else round(float(v), 4) for v in st["cell_mean_err"]]}
    x = synth.laplace_format_tensor()
    mask = O.sign_mask_from_seed(synth.sign_seed(4))
    for name, grid, scale, qmax in (("MXFP4", O.GRID_E2M1, O.SCALE_UE8M0_1x32, None),
                                    ("NVFP4", O.GRID_E2M1, O.SCALE_E4M3_1x16, 6.0),
                                    ("NVINT4", O.GRID_INT4, O.SCALE_E4M3_1x16, 7.0),
                                    ("IF4", O.GRID_IF4, O.SCALE_E4M3_1x16, 6.0)):
        cfg = O.OracleConfig(grid=grid, scale=scale, rht=1, sign_mask=mask)
        ts = None
        if qmax is not None:
            ts = float(np.float32(_tensor_amax(cfg, x)) / np.float32(qmax * 448.0))
        st = _stats(cfg, x, ts)
        row = {"nmse": round(st["nmse"], 6), "mse": round(st["mse"], 6), "sqnr_db": round(st["sqnr_db"], 2)}
        if grid == O.GRID_IF4:
            row["if4_fp4_fraction"] = round(st["if4_fp4_fraction"], 4)
        out["laplace_format_tensor %s" % name] = row
    print(json.dumps(out, indent=1))


if __name__ == "__main__":
    main()
