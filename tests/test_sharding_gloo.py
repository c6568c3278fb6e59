"""Two-rank (gloo, CPU) tests of the row-sharded host logic: each rank quantizes its row range
with the oracle as the compute step; the concatenated result must equal the unsharded one,
including the E4M3 tensor scale agreed by all-reduce(MAX), stochastic-rounding counters and the
summed statistics."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

WORLD = 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, port, case, out_dir):
    import torch.distributed as dist

    import oracle as O
    from block_scaled_bit_rht16_b200 import sharding, synth

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD)
    try:
        x = synth.small(77, 96, 256, "laplace")
        cfg = {
            "nvfp4": O.OracleConfig(grid=O.GRID_E2M1, scale=O.SCALE_E4M3_1x16, sign_mask=0x1234),
            "if4": O.OracleConfig(grid=O.GRID_IF4, scale=O.SCALE_E4M3_1x16, sign_mask=0x4321),
            "ufp4_sr": O.OracleConfig(grid=O.GRID_E1M2, round=O.ROUND_SR, sign_mask=0x0FF0, sr_seed=9),
        }[case]
        r0, r1 = sharding.row_range(x.shape[0], rank, WORLD, multiple=16)
        xs = np.ascontiguousarray(x[r0:r1])
        # the shard is quantized as a tensor of its own, as the library's call sees it: element
        # indices from 0, with the stochastic-rounding seed shifted to where its rows start
        from dataclasses import replace
        scfg = replace(cfg, sr_seed=sharding.shard_sr_seed(cfg.sr_seed, r0, x.shape[1]))
        steps = sharding.ShardSteps(
            tensor_scale=lambda: np.float32(O.tensor_amax(cfg, xs)) / np.float32(6.0 * 448.0),
            quantize=lambda alpha: O.quantize(scfg, xs, row0=0, tensor_scale=alpha, stats=True))
        res = sharding.quantize_rows_sharded(steps, cfg.scale == O.SCALE_E4M3_1x16)
        stats = sharding.global_stats_raw(res["stats_raw"])
        np.savez(os.path.join(out_dir, "r%d.npz" % rank), codes=res["codes"], scales=res["scales"],
                 alpha=np.float32(res["tensor_scale"] or 0.0), stats=stats, r0=r0, r1=r1)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("case", ["nvfp4", "if4", "ufp4_sr"])
def test_row_sharded_equals_unsharded(case, tmp_path):
    import oracle as O
    from block_scaled_bit_rht16_b200 import synth
    mp.start_processes(_worker, args=(_free_port(), case, str(tmp_path)), nprocs=WORLD,
                       start_method="spawn", join=True)
    parts = [np.load(os.path.join(tmp_path, "r%d.npz" % r)) for r in range(WORLD)]
    x = synth.small(77, 96, 256, "laplace")
    cfg = {
        "nvfp4": O.OracleConfig(grid=O.GRID_E2M1, scale=O.SCALE_E4M3_1x16, sign_mask=0x1234),
        "if4": O.OracleConfig(grid=O.GRID_IF4, scale=O.SCALE_E4M3_1x16, sign_mask=0x4321),
        "ufp4_sr": O.OracleConfig(grid=O.GRID_E1M2, round=O.ROUND_SR, sign_mask=0x0FF0, sr_seed=9),
    }[case]
    full = O.quantize(cfg, x, stats=True)
    assert [int(p["r0"]) for p in parts] == [0, 48] and int(parts[-1]["r1"]) == 96
    np.testing.assert_array_equal(np.concatenate([p["codes"] for p in parts]), full["codes"])
    np.testing.assert_array_equal(np.concatenate([p["scales"] for p in parts]), full["scales"])
    if full["tensor_scale"] is not None:
        assert all(p["alpha"] == np.float32(full["tensor_scale"]) for p in parts)
    for p in parts:
        np.testing.assert_allclose(p["stats"], full["stats_raw"], rtol=1e-12, atol=1e-12)


def test_row_range_partitions():
    from block_scaled_bit_rht16_b200 import sharding
    for rows, world, mult in [(96, 2, 16), (8192, 8, 16), (100, 3, 1), (16, 4, 16)]:
        spans = [sharding.row_range(rows, r, world, mult) for r in range(world)]
        assert spans[0][0] == 0 and spans[-1][1] == rows
        assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
        assert all(s[0] % mult == 0 for s in spans)
    with pytest.raises(ValueError):
        sharding.row_range(20, 0, 2, 16)


def test_shard_seed_reproduces_the_draws_of_every_row_range():
    # without any communication, a row range quantized on its own with the shifted seed gives
    # the rows of the whole tensor's result, in both counter streams and for ragged starts
    import oracle as O
    from dataclasses import replace
    from block_scaled_bit_rht16_b200 import sharding, synth
    x = synth.small(78, 40, 96, "normal")
    for stream in (0, 1):
        cfg = O.OracleConfig(grid=O.GRID_INT4, round=O.ROUND_SR, sign_mask=0x0F0F,
                             sr_seed=0xFFFF_FFFF_FFFF_FFF0, sr_stream=stream)
        full = O.quantize(cfg, x)["codes"]
        for r0 in (0, 1, 7, 39):
            part = O.quantize(replace(cfg, sr_seed=sharding.shard_sr_seed(cfg.sr_seed, r0, 96)),
                              np.ascontiguousarray(x[r0:]))["codes"]
            np.testing.assert_array_equal(part, full[r0:])
        # the unshifted seed does not: the shift is what makes the shard agree
        assert not np.array_equal(O.quantize(cfg, np.ascontiguousarray(x[7:]))["codes"], full[7:])
    with pytest.raises(ValueError):
        sharding.shard_sr_seed(1, 3, 6)
