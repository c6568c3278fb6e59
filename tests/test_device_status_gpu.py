"""The bounded waits of the bulk-copy pipeline: a deliberately starved wait runs out and
reports through the status word (no fault, no hang), and normal launches report nothing."""
import ctypes

import numpy as np
import pytest
import torch

import block_scaled_bit_rht16_b200 as fq
from block_scaled_bit_rht16_b200 import _lib, synth
from helpers import host, to_dev

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_and_cleared():
    fq.device_status(clear=True)
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert _lib.load().fp4q_check_wait_timeout(10_000_000, s) == 0     # 10 ms, nothing arrives
    assert fq.device_status() & 2
    assert fq.device_status(clear=True) & 2
    assert fq.device_status() == 0
    # the context is still usable: a normal launch works afterwards
    x = torch.ones((16, 64), dtype=torch.bfloat16, device="cuda")
    q = fq.rht_quantize(fq.Config(rht=0), x)
    torch.cuda.synchronize()
    assert (host(q.scales) == np.float32(1.0) / np.float32(3.5)).all()


def test_pipelined_launches_report_no_timeouts():
    fq.device_status(clear=True)
    x, w = synth.dense_linear_operands(rows=2048)
    t = to_dev(np.concatenate([x, w], axis=0))
    for grid in (fq.FP4Q_GRID_E1M2, fq.FP4Q_GRID_E2M1, fq.FP4Q_GRID_INT4):
        for _ in range(3):
            fq.rht_quantize(fq.Config(grid=grid, sign_mask=0x1234), t)
    torch.cuda.synchronize()
    assert fq.device_status() == 0
