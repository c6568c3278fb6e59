"""Tensors on either side of the row kernels' 32-bit offset limit.

Flat launches index blocks with 32-bit counters and elements as 16 * block in 32 bits, so they
take tensors of at most 2^28 blocks of 16 (2^32 elements); larger tensors take the 64-bit path.
A [65535, 65536] bf16 tensor (2^28 - 4096 blocks) runs flat with element offsets up to
2^32 - 65536; a [65537, 65536] tensor (2^28 + 4096 blocks) must take the 64-bit path, whose last
row starts exactly 2^32 elements in. Both are built from 61 distinct rows repeated, so the
oracle checks any row from its source row alone (and the whole tensor's amax is the source
rows' amax); rows at the start, at the 2^32-element boundary and at the end are compared with
the oracle.
"""
import numpy as np
import pytest

import oracle as O
import block_scaled_bit_rht16_b200 as fq
from block_scaled_bit_rht16_b200 import synth
from helpers import ocfg, to_dev, host

pytestmark = pytest.mark.gpu

COLS = 65536
SOURCE_ROWS = 61


def _tiled(base_dev, rows):
    import torch
    x = torch.empty((rows, COLS), dtype=torch.bfloat16, device="cuda")
    for r0 in range(0, rows, SOURCE_ROWS):
        n = min(SOURCE_ROWS, rows - r0)
        x[r0:r0 + n].copy_(base_dev[:n])
    return x


@pytest.mark.parametrize("rows", [65535, 65537])
@pytest.mark.parametrize("fmt", ["ufp4", "nvfp4"])
def test_rows_across_the_32_bit_element_offset(rows, fmt):
    import torch
    base = synth.small(91, SOURCE_ROWS, COLS, "t4")
    mask = fq.sign_mask_from_seed(synth.sign_seed(9))
    if fmt == "ufp4":   # the hot path: E1M2, rotation, FP32 scales, round to nearest
        cfg = fq.Config(grid=fq.FP4Q_GRID_E1M2, rht=1, sign_mask=mask)
    else:               # NVFP4 with the tensor scale computed: amax pass + E4M3 kernel
        cfg = fq.Config(grid=fq.FP4Q_GRID_E2M1, scale=fq.FP4Q_SCALE_E4M3_1x16_TENSOR, rht=1,
                        sign_mask=mask)
    x = _tiled(to_dev(base), rows)
    q = fq.rht_quantize(cfg, x)
    torch.cuda.synchronize()
    ref = O.quantize(ocfg(cfg), base)
    if fmt == "nvfp4":
        assert float(host(q.tensor_scale)[0]) == ref["tensor_scale"]
    boundary = (1 << 32) // COLS    # the row that starts 2^32 elements in
    for r in sorted({0, 1, boundary - 2, boundary - 1, boundary, rows - 2, rows - 1}):
        if r >= rows:
            continue
        src = r % SOURCE_ROWS
        np.testing.assert_array_equal(host(q.codes[r]), ref["codes"][src], err_msg="codes, row %d" % r)
        np.testing.assert_array_equal(host(q.scales[r]), ref["scales"][src], err_msg="scales, row %d" % r)
    del q, x
    torch.cuda.empty_cache()
