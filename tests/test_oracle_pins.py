"""Pins of the CPU oracle to facts outside itself (runs without a GPU).

Each test ties one oracle function to something the pages print, to a closed form, to a library
routine, to an invariant of the mathematics, or to brute force on tiny inputs, so that a
dropped term, a wrong sign or index, or a transposed operand fails at least one of them.
"""
import math
import os

import numpy as np
import pytest
import scipy.linalg
import torch

import oracle as O
from block_scaled_bit_rht16_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


GRID_IDS = {"E2M1": O.GRID_E2M1, "E1M2": O.GRID_E1M2, "INT4": O.GRID_INT4,
            "E2M1_MAX2": O.GRID_E2M1_MAX2}


# ------------------------------------------------------------------ number formats

def test_grids_match_printed_tables():
    for name, *vals in _golden_lines("grids.txt"):
        np.testing.assert_array_equal(O.grid_magnitudes(GRID_IDS[name]), np.array(vals, float))


def test_restricted_e2m1_grids_are_prefixes_of_e2m1():
    # the page's limits 4, 3, 2: the E2M1 magnitudes up to the limit, codes unchanged
    full = O.grid_magnitudes(O.GRID_E2M1)
    for grid, top in [(O.GRID_E2M1_MAX4, 4.0), (O.GRID_E2M1_MAX3, 3.0), (O.GRID_E2M1_MAX2, 2.0)]:
        g = O.grid_magnitudes(grid)
        np.testing.assert_array_equal(g, full[full <= top])
        # decoding is E2M1's for every code, also the unused ones
        for nib in range(16):
            assert O.decode_nibble(grid, nib) == O.decode_nibble(O.GRID_E2M1, nib)


def _restricted_rtne_brute(v, top):
    """Nearest value of {E2M1 magnitudes <= top}, ties to the even code, saturating; sign kept."""
    full = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    cand = [(c, m) for c, m in enumerate(full) if m <= top]
    a = abs(float(v))
    if a >= top:
        code = cand[-1][0]
    else:
        code = min(cand, key=lambda cm: (abs(a - cm[1]), cm[0] & 1))[0]
    return (8 if math.copysign(1.0, float(v)) < 0 else 0) | code


def test_restricted_e2m1_rtne_brute_force():
    vals = np.concatenate([np.arange(-8, 8.0001, 0.125), [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0],
                           np.random.default_rng(3).uniform(-7, 7, 2000)]).astype(np.float32)
    vals = np.concatenate([vals, -np.zeros(1, np.float32)])
    for grid, top in [(O.GRID_E2M1_MAX4, 4.0), (O.GRID_E2M1_MAX3, 3.0), (O.GRID_E2M1_MAX2, 2.0)]:
        got = O.round_rtne(grid, vals)
        want = np.array([_restricted_rtne_brute(v, top) for v in vals], np.uint8)
        np.testing.assert_array_equal(got, want)


def test_restricted_e2m1_block_scale_and_saturation():
    # FP32 1x16 scale s = RN(amax / top): in every nonzero block the largest element lands on
    # the top code, and no code above it is ever produced
    x = synth.small(17, 64, 128, "laplace")
    for grid, top, topcode in [(O.GRID_E2M1_MAX4, 4.0, 6), (O.GRID_E2M1_MAX3, 3.0, 5),
                               (O.GRID_E2M1_MAX2, 2.0, 4)]:
        cfg = O.OracleConfig(grid=grid, scale=O.SCALE_FP32_1x16, rht=0)
        out = O.quantize(cfg, x)
        codes = out["codes"]
        nib = np.stack([codes & 0xF, codes >> 4], axis=-1).reshape(x.shape[0], -1)
        assert int((nib & 7).max()) == topcode
        s = out["scales"].reshape(x.shape[0], -1)
        blocks_top = (nib & 7).reshape(x.shape[0], -1, 16).max(axis=-1)
        assert np.all(blocks_top[s > 0] == topcode)
    with pytest.raises(Exception):
        O.quantize(O.OracleConfig(grid=O.GRID_E2M1_MAX4, scale=O.SCALE_E4M3_1x16, rht=0), x)


def test_e1m2_grid_is_uniform_and_e2m1_is_not():
    g = O.grid_magnitudes(O.GRID_E1M2)
    assert np.all(np.diff(g) == 0.5)
    assert len(set(np.diff(O.grid_magnitudes(O.GRID_E2M1)))) > 1


def test_decode_nibble_sign_conventions():
    # sign-magnitude for the FP grids, two's complement for INT4 (readings R6)
    assert O.decode_nibble(O.GRID_E2M1, 0xF) == -6.0
    assert O.decode_nibble(O.GRID_E1M2, 0xF) == -3.5
    assert O.decode_nibble(O.GRID_E2M1, 0x8) == 0.0 and math.copysign(1, O.decode_nibble(O.GRID_E2M1, 0x8)) == -1
    assert O.decode_nibble(O.GRID_INT4, 0x9) == -7.0
    assert O.decode_nibble(O.GRID_INT4, 0xF) == -1.0


def _e2m1_by_exponent(a):
    """IEEE-style rounding of |v| onto E2M1 written from the format's exponent/step structure
    (independent of the oracle's nearest-point search): step 0.5 below 2, 1 in [2, 4),
    2 in [4, 8); round-half-even on the step count; saturate at 6."""
    a = np.asarray(a, dtype=np.float64)
    step = np.where(a < 2, 0.5, np.where(a < 4, 1.0, 2.0))
    q = np.rint(a / step) * step
    return np.minimum(q, 6.0)


def _value_of(grid, codes):
    return np.array([O.decode_nibble(grid, int(c)) for c in range(16)])[codes]


@pytest.mark.parametrize("grid", [O.GRID_E2M1, O.GRID_E1M2, O.GRID_INT4])
def test_rtne_against_independent_formula(grid):
    # every float in [0, 9] with a 2^-12 stride, plus dense neighbourhoods of every midpoint
    rng = np.random.default_rng(7)
    base = np.arange(0, 9 * 4096 + 1, dtype=np.float64) / 4096
    g = O.grid_magnitudes(grid)
    mids = (g[1:] + g[:-1]) / 2
    near = [np.nextafter(np.float32(m), np.float32(np.inf * s)) for m in mids for s in (-1, 1)]
    u = rng.integers(0, 0x41100000, size=200_000).astype(np.uint32).view(np.float32)
    v = np.concatenate([base.astype(np.float32), np.float32(mids), np.float32(near), u])
    v = np.concatenate([v, -v])
    got = _value_of(grid, O.round_rtne(grid, v))
    a = np.abs(v.astype(np.float64))
    if grid == O.GRID_E2M1:
        want = _e2m1_by_exponent(a)
    elif grid == O.GRID_E1M2:
        want = np.minimum(np.rint(2 * a) / 2, 3.5)     # numpy rint is round-half-even
    else:
        want = np.minimum(np.rint(a), 7.0)
    want = np.copysign(want, v)
    np.testing.assert_array_equal(np.abs(got), np.abs(want))
    nz = want != 0
    np.testing.assert_array_equal(np.sign(got[nz]), np.sign(want[nz]))


@pytest.mark.parametrize("grid", [O.GRID_E2M1, O.GRID_E1M2, O.GRID_INT4])
def test_rtne_saturates_far_above_qmax(grid):
    # the nearest point to anything above the largest magnitude is that magnitude
    g = O.grid_magnitudes(grid)
    v = np.float32([g[7] * 1.01, 1e10, 2.0 ** 60, 3e38, -1e30, -(2.0 ** 100)])
    got = _value_of(grid, O.round_rtne(grid, v))
    np.testing.assert_array_equal(got, np.copysign(g[7], v))


def test_rtne_tie_table_reading():
    # reading R5: ties go to the even code
    v = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32)
    np.testing.assert_array_equal(_value_of(O.GRID_E2M1, O.round_rtne(O.GRID_E2M1, v)),
                                  [0, 1, 1, 2, 2, 4, 4])
    v = np.array([0.25, 0.75, 1.25, 1.75, 3.25], np.float32)
    np.testing.assert_array_equal(_value_of(O.GRID_E1M2, O.round_rtne(O.GRID_E1M2, v)),
                                  [0, 1, 1, 2, 3])


def test_negative_zero_codes():
    # R6: a negative value that rounds to zero keeps its sign on the sign-magnitude grids
    assert O.round_rtne(O.GRID_E2M1, np.float32([-0.1]))[0] == 0x8
    assert O.round_rtne(O.GRID_E1M2, np.float32([-0.0]))[0] == 0x8
    assert O.round_rtne(O.GRID_INT4, np.float32([-0.1]))[0] == 0x0


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.standard_normal(200_000).astype(np.float32),
                        (rng.integers(0, 2**31, 200_000).astype(np.uint32)).view(np.float32)])
    x = x[np.isfinite(x) & (np.abs(x) < 3e38)]
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(O.f32_to_bf16(x), ref)


def test_e4m3_encoder_matches_torch_in_range():
    rng = np.random.default_rng(11)
    x = np.concatenate([rng.uniform(0, 460, 100_000), 2.0 ** rng.uniform(-12, 8.8, 100_000),
                        [0.0, 2**-10, 1.5 * 2**-10, 2**-9, 448.0, 463.9]]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(O.e4m3_encode(x), ref)


def test_e4m3_every_code_midpoint_and_its_neighbours():
    # the decode table of all 127 finite non-negative codes equals torch's float8_e4m3fn values,
    # and at every midpoint between adjacent values (a tie: to the even code) and at the FP32
    # neighbours on either side of it the encoder agrees with torch's conversion
    codes = torch.arange(127, dtype=torch.uint8)
    vals = codes.view(torch.float8_e4m3fn).to(torch.float32).numpy()
    np.testing.assert_array_equal(np.array([O.e4m3_decode(c) for c in range(127)], np.float32), vals)
    mids = ((vals[1:].astype(np.float64) + vals[:-1]) / 2).astype(np.float32)
    assert np.all(mids.astype(np.float64) == (vals[1:].astype(np.float64) + vals[:-1]) / 2)  # exact
    probe = np.concatenate([mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(1e9)),
                            vals]).astype(np.float32)
    ref = torch.from_numpy(probe).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(O.e4m3_encode(probe), ref)


def test_e4m3_saturates_and_decodes():
    assert O.e4m3_encode(np.float32([448.0, 500.0, 1e30, np.inf])).tolist() == [0x7E] * 4
    assert O.e4m3_decode(0x7E) == 448.0
    assert O.e4m3_decode(0x01) == 2.0 ** -9
    ref = torch.arange(0, 0x7F, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    np.testing.assert_array_equal([O.e4m3_decode(b) for b in range(0x7F)], ref)


def test_format_limits_table():
    # IF4 page section 2.2 table, with tensor scale 1
    lim = {r[0]: (eval(r[1].replace("^", "**")), eval(r[2].replace("^", "**")))
           for r in _golden_lines("format_limits.txt")}
    d8max, d8min = O.e4m3_decode(0x7E), O.e4m3_decode(0x01)
    g_fp, g_int = O.grid_magnitudes(O.GRID_E2M1), O.grid_magnitudes(O.GRID_INT4)
    assert (g_fp[7] * d8max, g_fp[1] * d8min) == lim["NVFP4"]
    assert (g_int[7] * d8max, g_int[1] * d8min) == lim["NVINT4"]
    assert (g_fp[7] * d8max, g_fp[1] * d8min) == lim["IF4"]
    # UE8M0 codes 0..254 decode to 2^(code-127)
    assert (g_fp[7] * 2.0 ** (254 - 127), g_fp[1] * 2.0 ** (0 - 127)) == lim["MXFP4"]


def test_mx_exponent_rule():
    rng = np.random.default_rng(5)
    for a in np.concatenate([2.0 ** rng.uniform(-120, 120, 2000), 2.0 ** np.arange(-120, 121)]):
        a = np.float32(a)
        e = O.mx_exponent(a)
        assert 4.0 <= float(a) * 2.0 ** -e < 8.0      # amax * 2^-e lands in [4, 8)
    assert O.mx_exponent(np.float32(2.0 ** -130)) == -127   # clamped
    assert O.mx_exponent(np.float32(0.0)) == -127


# ------------------------------------------------------------------ rotation

def test_sylvester_matches_scipy_and_is_orthogonal():
    h = O.sylvester_h16()
    np.testing.assert_array_equal(h, scipy.linalg.hadamard(16))
    np.testing.assert_array_equal(h @ h.T, 16 * np.eye(16, dtype=np.int32))
    # closed form of the natural (Sylvester) order
    i, j = np.meshgrid(np.arange(16), np.arange(16), indexing="ij")
    pop = np.vectorize(lambda t: bin(t).count("1"))(i & j)
    np.testing.assert_array_equal(h, (-1) ** pop)


def test_butterfly_equals_matvec_on_unit_and_integer_vectors():
    h = scipy.linalg.hadamard(16).astype(np.float64)
    for j in range(16):
        e = np.zeros(16, np.float32)
        e[j] = 1.0
        np.testing.assert_array_equal(O.rht16(e, 0), (h[:, j] / 4).astype(np.float32))
        # the sign mask bit j negates exactly input j
        np.testing.assert_array_equal(O.rht16(e, 1 << j), (-h[:, j] / 4).astype(np.float32))
    rng = np.random.default_rng(1)
    for _ in range(500):
        x = rng.integers(-1000, 1001, 16).astype(np.float32)
        mask = int(rng.integers(0, 1 << 16))
        d = np.array([-1.0 if (mask >> k) & 1 else 1.0 for k in range(16)])
        want = (h @ (d * x.astype(np.float64))) / 4
        np.testing.assert_array_equal(O.rht16(x, mask), want.astype(np.float32))


def test_rht_invertible_and_norm_preserving():
    rng = np.random.default_rng(2)
    for _ in range(500):
        x = rng.integers(-8, 9, 16).astype(np.float32)
        mask = int(rng.integers(0, 1 << 16))
        y = O.rht16(x, mask)
        np.testing.assert_array_equal(O.inverse_rht16(y, mask), x)
        assert float(np.sum(y.astype(np.float64) ** 2)) == float(np.sum(x.astype(np.float64) ** 2))
    for _ in range(500):
        x = rng.standard_normal(16).astype(np.float32)
        mask = int(rng.integers(0, 1 << 16))
        y = O.rht16(x, mask)
        nx = np.linalg.norm(x.astype(np.float64))
        assert abs(np.linalg.norm(y.astype(np.float64)) - nx) <= 8 * 2.0 ** -24 * nx
        np.testing.assert_allclose(O.inverse_rht16(y, mask), x, rtol=0, atol=8 * 2.0 ** -24 * nx)


# ------------------------------------------------------------------ stochastic rounding

def test_splitmix64_published_vectors():
    outs = [int(ln[0], 16) for ln in _golden_lines("splitmix64.txt")]
    gamma = 0x9E3779B97F4A7C15
    assert [O.splitmix64((k * gamma) % 2**64) for k in range(3)] == outs


def test_sr_probability_exact_by_enumeration():
    # P(round up) = ceil(frac * 2^16) / 2^16, counted over every draw u (r = u * 2^-16)
    k = np.arange(1 << 16, dtype=np.uint32)
    for grid, v in [(O.GRID_E1M2, 1.3), (O.GRID_E1M2, 0.0001), (O.GRID_E2M1, 2.7),
                    (O.GRID_E2M1, 4.5), (O.GRID_INT4, 3.999), (O.GRID_E1M2, 3.4999),
                    (O.GRID_E2M1, 0.74), (O.GRID_INT4, 6.0000005), (O.GRID_E1M2, 1e-30),
                    (O.GRID_E2M1_MAX4, 3.3), (O.GRID_E2M1_MAX3, 2.7), (O.GRID_E2M1_MAX2, 1.9)]:
        v32 = np.float32(v)
        g = O.grid_magnitudes(grid)
        lo = g[np.searchsorted(g, v32, side="right") - 1]
        hi = g[np.searchsorted(g, v32, side="right")]
        frac = (float(v32) - lo) / (hi - lo)
        codes = O.round_sr(grid, np.full(k.shape, v32), k)
        ups = int(np.count_nonzero(_value_of(grid, codes) == hi))
        assert ups == math.ceil(frac * 2**16), (grid, v)
        assert np.all((_value_of(grid, codes) == hi) | (_value_of(grid, codes) == lo))


def test_sr_keeps_grid_points_and_is_unbiased():
    rng = np.random.default_rng(9)
    for grid in (O.GRID_E1M2, O.GRID_E2M1, O.GRID_INT4):
        g = O.grid_magnitudes(grid)
        u = rng.integers(0, 2**32, size=(8, 4096), dtype=np.uint64).astype(np.uint32)
        u[0, :] = 0                    # r = 0: a grid point (frac = 0) must still stay put
        on = np.repeat(np.concatenate([g, -g]).astype(np.float32), 512)[: u.size]
        np.testing.assert_array_equal(_value_of(grid, O.round_sr(grid, on, u.reshape(-1)[: on.size])), on)
    n = 1_000_000
    bits = np.array([O.sr_bits(0x5A5A0003, 0, i) for i in range(n)], dtype=np.uint32)
    for v in (0.3, 1.1, 2.2, 3.37):
        vals = _value_of(O.GRID_E1M2, O.round_sr(O.GRID_E1M2, np.full(n, np.float32(v)), bits))
        sigma = 0.5 * math.sqrt(((v % 0.5) / 0.5) * (1 - (v % 0.5) / 0.5) / n)
        assert abs(vals.mean() - float(np.float32(v))) < 4 * sigma + 1e-12


def test_sr_bits_lanes_and_streams():
    # elements 4k .. 4k+3 take the four 16-bit lanes (low lane first) of output k of the
    # SplitMix64 stream seeded with seed ^ (stream << 63): the finalizer of state
    # seed' + (k+1) * gamma, stepped here one gamma at a time from the seed
    gamma, mask = 0x9E3779B97F4A7C15, 2**64 - 1
    for seed, k in ((1, 0), (1, 250), (0x5A5A0003, 2**38 + 5)):
        for stream in (0, 1):
            state = seed ^ (stream << 63)
            if k < 1000:
                for _ in range(k):
                    state = (state + gamma) & mask
            else:
                state = (state + k * gamma) & mask
            h = O.splitmix64(state)
            lanes = [(h >> (16 * l)) & 0xFFFF for l in range(4)]
            assert [O.sr_bits(seed, stream, 4 * k + l) for l in range(4)] == lanes
    assert O.sr_bits(1, 1, 1000) != O.sr_bits(1, 0, 1000)
    bits = np.array([O.sr_bits(123, 0, i) for i in range(200_000)], dtype=np.uint64)
    assert int(bits.max()) < 2**16
    for b in range(16):
        frac = np.mean((bits >> np.uint64(b)) & np.uint64(1))
        assert abs(frac - 0.5) < 0.01


# ------------------------------------------------------------------ shrinkage bias

def _cell_lattice(grid, q):
    """Midpoint lattice of step 1/16 over the rounding cell of q (exact in bfloat16 here)."""
    g = O.grid_magnitudes(grid)
    c = int(np.where(g == q)[0][0])
    left = (g[c] - g[c - 1]) / 2 if c > 0 else 0.0
    right = (g[c + 1] - g[c]) / 2 if c < len(g) - 1 else 0.0
    h = 1.0 / 16
    n = int(round((left + right) / h))
    return q - left + (np.arange(n) + 0.5) * h, left, right


def _bias_blocks(grid, q):
    """Blocks of 16 with element 0 = qmax (so the FP32 scale is exactly 1 and v = y) and 15
    points of the cell lattice of q (the lattice repeated 15 times, so the mean is exact)."""
    lat, _, _ = _cell_lattice(grid, q)
    qmax = O.grid_magnitudes(grid)[-1]
    blocks = np.tile(lat, 15).reshape(-1, 15)
    x = np.concatenate([np.full((blocks.shape[0], 1), qmax), blocks], axis=1).astype(np.float32)
    return synth.to_bf16_bits(x), x


@pytest.mark.parametrize("row", _golden_lines("shrinkage_bias.txt"))
def test_printed_shrinkage_bias(row):
    name, q, ln, rn, lw, rw, expected = row
    grid, q = GRID_IDS[name], float(q)
    lat, left, right = _cell_lattice(grid, q)
    assert (left, right) == (float(lw), float(rw))
    assert (left - right) / 2 == float(expected)
    bits, x = _bias_blocks(grid, q)
    assert np.array_equal(synth.bf16_bits_to_f32(bits), x)     # lattice exact in bfloat16
    cfg = O.OracleConfig(grid=grid, rht=0)
    st = O.finalize_stats(O.quantize(cfg, bits, stats=True)["stats_raw"])
    c = int(np.where(O.grid_magnitudes(grid) == q)[0][0])
    assert st["cell_mean_err"][c] == pytest.approx(float(expected), abs=1e-12)


@pytest.mark.parametrize("grid", [O.GRID_E2M1, O.GRID_E1M2, O.GRID_INT4])
def test_shrinkage_bias_closed_form_every_cell(grid):
    g = O.grid_magnitudes(grid)
    for c in range(1, 7):
        bits, _ = _bias_blocks(grid, g[c])
        st = O.finalize_stats(O.quantize(O.OracleConfig(grid=grid, rht=0), bits, stats=True)["stats_raw"])
        left, right = (g[c] - g[c - 1]) / 2, (g[c + 1] - g[c]) / 2
        assert st["cell_mean_err"][c] == pytest.approx((left - right) / 2, abs=1e-9)
        if grid != O.GRID_E2M1:
            assert st["cell_mean_err"][c] == pytest.approx(0.0, abs=1e-9)


@pytest.mark.parametrize("grid", [O.GRID_E2M1_MAX4, O.GRID_E2M1_MAX3, O.GRID_E2M1_MAX2])
def test_shrinkage_bias_closed_form_restricted_e2m1(grid):
    # interior cells (L - R) / 2 as for E2M1; the new top cell is clipped on the right (values
    # never exceed the limit), so its lattice has mean signed error +L / 2 -- diluted to
    # 15/16 of that by each block's scale-setting element, which sits at the limit with error 0
    g = O.grid_magnitudes(grid)
    top = len(g) - 1
    for c in range(1, len(g)):
        bits, _ = _bias_blocks(grid, g[c])
        st = O.finalize_stats(O.quantize(O.OracleConfig(grid=grid, rht=0), bits, stats=True)["stats_raw"])
        left = (g[c] - g[c - 1]) / 2
        if c < top:
            want = (left - (g[c + 1] - g[c]) / 2) / 2
        else:
            want = (15.0 / 16.0) * left / 2
        assert st["cell_mean_err"][c] == pytest.approx(want, abs=1e-9)


# ------------------------------------------------------------------ quantizer invariants

def _signed_grid(grid):
    g = O.grid_magnitudes(grid)
    return np.unique(np.concatenate([-g, g]))


@pytest.mark.parametrize("grid", [O.GRID_E2M1, O.GRID_E1M2, O.GRID_INT4])
@pytest.mark.parametrize("rht", [0, 1])
def test_fp32_scale_nearest_point_and_qmax(grid, rht):
    x = synth.small(21, 64, 256, "t4")
    cfg = O.OracleConfig(grid=grid, rht=rht, sign_mask=0xA5C3)
    r = O.quantize(cfg, x, dequant=True)
    codes, s = r["codes"], r["scales"]
    nib = np.stack([codes & 0xF, codes >> 4], axis=-1).reshape(64, 256)
    q = _value_of(grid, nib)
    xf = synth.bf16_bits_to_f32(x)
    y = np.stack([O.rht16(b, 0xA5C3) for b in xf.reshape(-1, 16)]).reshape(64, 256) if rht else xf
    yb = y.reshape(64, 16, 16)
    amax = np.abs(yb).max(-1)
    qmax = O.grid_magnitudes(grid)[7]
    np.testing.assert_array_equal(s, (amax / np.float32(qmax)).astype(np.float32))
    v = (yb / s[..., None]).astype(np.float64)
    sg = _signed_grid(grid)
    dist = np.abs(v[..., None] - sg).min(-1)
    np.testing.assert_array_equal(np.abs(v - q.reshape(v.shape)), dist)    # nearest point
    assert np.all(np.abs(q.reshape(v.shape)).max(-1) == qmax)             # qmax is reached
    xhat = (q.reshape(v.shape) * s[..., None]).astype(np.float32)
    half = {O.GRID_E2M1: 1.0, O.GRID_E1M2: 0.25, O.GRID_INT4: 0.5}[grid]
    assert np.all(np.abs(xhat - yb) <= half * s[..., None] * (1 + 1e-6))


def test_e1m2_and_int4_share_magnitude_codes():
    x = synth.small(33, 128, 512, "laplace")
    a = O.quantize(O.OracleConfig(grid=O.GRID_E1M2, sign_mask=0x1234), x)
    b = O.quantize(O.OracleConfig(grid=O.GRID_INT4, sign_mask=0x1234), x)
    na = np.stack([a["codes"] & 0xF, a["codes"] >> 4], -1)
    nb = np.stack([b["codes"] & 0xF, b["codes"] >> 4], -1)
    np.testing.assert_array_equal(np.abs(_value_of(O.GRID_E1M2, na)) * 2,
                                  np.abs(_value_of(O.GRID_INT4, nb)))
    np.testing.assert_array_equal(a["scales"], b["scales"] * 2)   # RN(A/3.5) = 2 RN(A/7)


def test_nibble_order_and_packing():
    # R7: element 2j in the low nibble of byte j; s = 1 because the block holds 6 = qmax
    vals = np.array([6, 0.5, -1, 0, 2, -3, 4, 1.5, -6, 0, 0, 0, 0, 0, 1, -0.5], np.float32)
    r = O.quantize(O.OracleConfig(grid=O.GRID_E2M1, rht=0), synth.to_bf16_bits(vals[None]))
    assert r["scales"][0, 0] == 1.0
    assert r["codes"][0].tolist() == [0x17, 0x0A, 0xD4, 0x36, 0x0F, 0x00, 0x00, 0x92]


def test_zero_block_encodes_zero():
    x = np.zeros((2, 32), np.uint16)
    x[1, :16] = 0x8000          # -0.0
    for grid in (O.GRID_E2M1, O.GRID_E1M2, O.GRID_INT4):
        r = O.quantize(O.OracleConfig(grid=grid, sign_mask=0xFFFF), x, dequant=True, stats=True)
        assert not r["codes"].any() and not r["scales"].any() and not r["dequant"].any()


def test_dequantize_round_trip_and_inverse_rotation():
    x = synth.small(44, 32, 128, "normal")
    for cfg in [O.OracleConfig(grid=O.GRID_E1M2, sign_mask=0x0F0F),
                O.OracleConfig(grid=O.GRID_E2M1, scale=O.SCALE_E4M3_1x16, sign_mask=0x0F0F),
                O.OracleConfig(grid=O.GRID_IF4, scale=O.SCALE_E4M3_1x16, sign_mask=0x0F0F),
                O.OracleConfig(grid=O.GRID_E2M1, scale=O.SCALE_UE8M0_1x32, sign_mask=0x0F0F)]:
        r = O.quantize(cfg, x, dequant=True)
        d = O.dequantize(cfg, r["codes"], r["scales"], r["tensor_scale"], 32, 128)
        np.testing.assert_array_equal(d, r["dequant"])
        back = synth.bf16_bits_to_f32(O.dequantize(cfg, r["codes"], r["scales"], r["tensor_scale"],
                                                   32, 128, inverse_rht=True))
        xf = synth.bf16_bits_to_f32(x)
        assert np.linalg.norm(back - xf) < 0.2 * np.linalg.norm(xf)


def test_rht16_rows_matches_blockwise_rotation():
    x = synth.small(45, 8, 64, "normal")
    yf, yb = O.rht16_rows(x, 0x5555)
    xf = synth.bf16_bits_to_f32(x)
    want = np.stack([O.rht16(b, 0x5555) for b in xf.reshape(-1, 16)]).reshape(8, 64)
    np.testing.assert_array_equal(yf, want)
    np.testing.assert_array_equal(yb, O.f32_to_bf16(want))


# ------------------------------------------------------------------ NV / MX / IF4 scales

def test_nv_scales_follow_the_tensor_amax():
    x = synth.small(51, 64, 320, "laplace")
    cfg = O.OracleConfig(grid=O.GRID_E2M1, scale=O.SCALE_E4M3_1x16, sign_mask=0x3C3C)
    r = O.quantize(cfg, x, dequant=True)
    A = O.tensor_amax(cfg, x)
    # A is the largest magnitude of the rotated tensor, also when that element is negative
    yall = np.stack([O.rht16(b, 0x3C3C) for b in synth.bf16_bits_to_f32(x).reshape(-1, 16)])
    assert A == np.abs(yall).max()
    neg = synth.bf16_bits_to_f32(x).copy()
    neg[3, 17] = -1000.0
    ny = np.stack([O.rht16(b, 0x3C3C) for b in neg.reshape(-1, 16)])
    assert ny.max() < -ny.min()
    assert O.tensor_amax(cfg, synth.to_bf16_bits(neg)) == np.abs(ny).max()
    assert r["tensor_scale"] == np.float32(np.float32(A) / np.float32(6 * 448))
    assert r["scales"].max() == 0x7E                       # the block holding A gets 448
    assert np.all(r["scales"] <= 0x7E)
    xh = np.abs(synth.bf16_bits_to_f32(r["dequant"])).max()
    assert abs(xh - A) <= A * 2 ** -7                       # largest dequant value ~ A
    # NVINT4: same two-level rule with 7 in place of 6 (reading R9)
    c4 = O.OracleConfig(grid=O.GRID_INT4, scale=O.SCALE_E4M3_1x16, sign_mask=0x3C3C)
    r4 = O.quantize(c4, x)
    assert r4["tensor_scale"] == np.float32(np.float32(A) / np.float32(7 * 448))
    # every block's scale maps its own amax onto qmax: E4M3 keeps 3 mantissa bits, so in its
    # normal range RNE moves the block scale by at most 2^-4 relative, and amax_b / s lies in
    # qmax * [1/(1 + 2^-4), 1/(1 - 2^-4)] (IF4 page, section 3.2: the block scale is amax_b
    # over qmax in units of the tensor scale); blocks that saturate at 448 or fall below
    # E4M3's normal range are left out
    xf = synth.bf16_bits_to_f32(x).reshape(-1, 16)
    amax_b = np.abs(np.stack([O.rht16(b, 0x3C3C) for b in xf])).max(-1).astype(np.float64)
    dec = np.array([O.e4m3_decode(b) for b in range(128)], np.float64)
    for res, qmax in ((r, 6.0), (r4, 7.0)):
        d8 = dec[res["scales"].reshape(-1)]
        s_b = d8 * float(res["tensor_scale"])
        ok = (d8 >= 2.0 ** -6) & (d8 < 448)
        assert ok.sum() > 500
        ratio = amax_b[ok] / s_b[ok]
        assert np.all((ratio >= qmax / (1 + 2 ** -4) * (1 - 1e-6)) & (ratio <= qmax / (1 - 2 ** -4) * (1 + 1e-6)))


def test_mx_block_scale_powers_of_two():
    x = synth.small(52, 16, 256, "laplace", 3.0)
    cfg = O.OracleConfig(grid=O.GRID_E2M1, scale=O.SCALE_UE8M0_1x32, sign_mask=0x7777)
    r = O.quantize(cfg, x)
    xf = synth.bf16_bits_to_f32(x).reshape(-1, 16)
    y = np.stack([O.rht16(b, 0x7777) for b in xf]).reshape(16, 8, 32)
    amax = np.abs(y).max(-1)
    e = r["scales"].astype(np.int32) - 127
    assert np.all((amax * 2.0 ** -e >= 4) & (amax * 2.0 ** -e < 8))


def _nib(codes):
    return np.stack([codes & 0xF, codes >> 4], -1).reshape(codes.shape[0], -1)


def test_if4_choice_properties():
    x = synth.small(61, 256, 256, "uniform")
    mask = 0x0F33
    nv = O.quantize(O.OracleConfig(grid=O.GRID_E2M1, scale=O.SCALE_E4M3_1x16, sign_mask=mask), x, dequant=True)
    i4 = O.quantize(O.OracleConfig(grid=O.GRID_IF4, scale=O.SCALE_E4M3_1x16, sign_mask=mask), x, dequant=True)
    assert nv["tensor_scale"] == i4["tensor_scale"]
    np.testing.assert_array_equal(nv["scales"], i4["scales"] & 0x7F)       # same E4M3 magnitude
    xf = synth.bf16_bits_to_f32(x).reshape(-1, 16)
    y = np.stack([O.rht16(b, mask) for b in xf]).reshape(256, 16, 16).astype(np.float64)

    alpha = np.float32(nv["tensor_scale"])
    s = (np.array([O.e4m3_decode(b) for b in range(128)], np.float32)[nv["scales"]] * alpha)
    v = (y.astype(np.float32) / s[..., None]).astype(np.float64)

    def sse(r, if4):
        nib = _nib(r["codes"]).reshape(256, 16, 16)
        val = _value_of(O.GRID_E2M1, nib)
        if if4:
            intb = (r["scales"] >> 7).astype(bool)
            k = _value_of(O.GRID_INT4, nib)
            val = np.where(intb[..., None], (k * np.float32(6 / 7)).astype(np.float32), val)
        return ((val - v) ** 2).sum(-1)
    # the adaptive choice is never worse than plain NVFP4, in scaled units, up to FP32 summation
    assert np.all(sse(i4, True) <= sse(nv, False) * (1 + 1e-5) + 1e-30)
    flag = (i4["scales"] >> 7).astype(bool)
    assert 0 < flag.mean() < 1
    # FP4 blocks carry exactly the NVFP4 codes
    fp = ~flag
    n_nv, n_i4 = _nib(nv["codes"]).reshape(256, 16, 16), _nib(i4["codes"]).reshape(256, 16, 16)
    np.testing.assert_array_equal(n_nv[fp], n_i4[fp])


def test_if4_grid_and_int_lattice_blocks():
    # a block whose scaled values lie on the E2M1 grid keeps FP4 (zero error, ties to FP4)
    on_fp = np.array([6, 4, 3, 2, 1.5, 1, 0.5, 0, -6, -4, -3, -2, -1.5, -1, -0.5, 0], np.float32)
    # a block on the INT4 * 6/7 lattice (k = 0..7) prefers INT4
    on_int = np.array([k * 6 / 7 for k in range(8)] * 2, np.float32) * np.float32([1, -1] * 8)
    x = synth.to_bf16_bits(np.stack([on_fp, on_int]) * np.float32(0.75))
    cfg = O.OracleConfig(grid=O.GRID_IF4, scale=O.SCALE_E4M3_1x16, rht=0)
    r = O.quantize(cfg, x, tensor_scale=np.float32(0.75) * np.float32(6) / np.float32(6 * 448) * 448 / 448)
    flags = (r["scales"][:, 0] >> 7).tolist()
    assert flags == [0, 1]
    # INT4 code 7 dequantizes to 7 * RN(6/7) ~ 6 in scaled units
    assert abs(7 * np.float32(6 / 7) - 6) < 1e-6


def _if4_exact_int(y, s):
    """The IF4 page's INT4 candidate (section 3.1.1) in exact arithmetic: the value times 7/6
    over the block scale, rounded to the nearest integer (halves to even), limited to +-7."""
    from fractions import Fraction
    k = round(Fraction(float(y)) * 7 / (6 * Fraction(float(s))))
    return max(-7, min(7, k))


def _int4_nibbles(codes, n):
    nib = _nib(codes).reshape(-1)[:n].astype(np.int64)
    return np.where(nib >= 8, nib - 16, nib)


def test_if4_worked_example_int4_block():
    # IF4 page, section 3.1.1: an INT4 block multiplies its values by 7/6 before rounding to
    # integers and dequantizes integer * scale * 6/7; section 3.2: the block keeps INT4 when its
    # error is the smaller one, flagged in the scale byte's top bit.
    # The block: 6, 3, -1.2, 0.4 (INT4 7, 4, -1, 0; 3 * 7/6 = 3.5 is a tie that goes to the even
    # 4) and twelve values near k * 6/7, which E2M1 represents poorly and INT4 * 6/7 well.
    head = [6.0, 3.0, -1.2, 0.4]
    tail = [k * 6 / 7 * sg for k, sg in zip([6, 3, 5, 2, 1, 4] * 2, [1, -1] * 6)]
    x = synth.to_bf16_bits(np.array([head + tail], np.float32))
    y = synth.bf16_bits_to_f32(x)[0]
    # tensor scale 2^-8 and block amax 6: Delta = 6 / (2^-8 * 6) = 256, an E4M3 value, so the
    # block scale is s = 256 * 2^-8 = 1 exactly
    cfg = O.OracleConfig(grid=O.GRID_IF4, scale=O.SCALE_E4M3_1x16, rht=0)
    r = O.quantize(cfg, x, tensor_scale=np.float32(2.0 ** -8), dequant=True)
    sbyte = int(r["scales"][0, 0])
    assert sbyte >> 7 == 1, "the block must take INT4"
    assert O.e4m3_decode(sbyte & 0x7F) == 256.0
    k = _int4_nibbles(r["codes"], 16)
    assert k[:4].tolist() == [7, 4, -1, 0]
    assert k.tolist() == [_if4_exact_int(v, 1.0) for v in y]
    # dequantized: integer * scale * 6/7 (bf16 output; the FP32 products differ from the exact
    # ones by an ulp at most)
    got = synth.bf16_bits_to_f32(r["dequant"][0]).astype(np.float64)
    np.testing.assert_allclose(got, k * 6 / 7, rtol=2.0 ** -8, atol=0)
    # the printed coefficient table: FP4 x INT4 blocks carry 6/7, INT4 x INT4 blocks (6/7)^2
    coeffs = {row[0]: eval(row[1]) for row in _golden_lines("if4_coefficients.txt")}
    assert coeffs["FP4xINT4"] == pytest.approx(6 / 7) and coeffs["INT4xINT4"] == pytest.approx(36 / 49)


def test_if4_int_candidate_follows_the_page_rule_up_to_rounding():
    # every INT4 block the oracle emits has the codes of the page's rule round(y * 7/6 / s) in
    # exact arithmetic, except for values within FP32 rounding of a half-integer, where the
    # order of the two FP32 operations decides (the oracle scales y by s first, then by 7/6)
    from fractions import Fraction
    x = synth.small(91, 128, 256, "laplace")
    cfg = O.OracleConfig(grid=O.GRID_IF4, scale=O.SCALE_E4M3_1x16, rht=0)
    r = O.quantize(cfg, x)
    alpha = np.float32(r["tensor_scale"])
    e4 = np.array([O.e4m3_decode(b) for b in range(128)], np.float32)
    s = (e4[r["scales"] & 0x7F] * alpha).astype(np.float32)      # FP32 block scales
    yb = synth.bf16_bits_to_f32(x).reshape(128, 16, 16)
    flag = (r["scales"] >> 7).astype(bool)
    kk = _int4_nibbles(r["codes"], x.size).reshape(128, 16, 16)
    checked = near = 0
    for i, j in zip(*np.nonzero(flag)):
        for e in range(16):
            t = Fraction(float(yb[i, j, e])) * 7 / (6 * Fraction(float(s[i, j])))
            frac = abs(t) - math.floor(abs(t))
            if abs(frac - Fraction(1, 2)) < Fraction(1, 2 ** 20) and abs(t) < 7:
                near += 1
                continue
            assert kk[i, j, e] == _if4_exact_int(yb[i, j, e], s[i, j])
            checked += 1
    assert checked > 10000 and near <= checked // 1000


# ------------------------------------------------------------------ statistics

def test_stats_on_grid_input_and_direct_formulas():
    on = np.array([6, 4, 3, 2, 1.5, 1, 0.5, 0] * 2, np.float32)
    st = O.finalize_stats(O.quantize(O.OracleConfig(grid=O.GRID_E2M1, rht=0),
                                     synth.to_bf16_bits(on[None]), stats=True)["stats_raw"])
    assert st["sqnr_db"] == math.inf and st["alpha"] == 1.0
    x = synth.small(71, 64, 128, "normal")
    cfg = O.OracleConfig(grid=O.GRID_E1M2, sign_mask=0x1111)
    r = O.quantize(cfg, x, dequant=True, stats=True)
    st = O.finalize_stats(r["stats_raw"])
    xf = synth.bf16_bits_to_f32(x).reshape(-1, 16)
    y = np.stack([O.rht16(b, 0x1111) for b in xf]).reshape(-1).astype(np.float64)
    xh = synth.bf16_bits_to_f32(r["dequant"]).reshape(-1).astype(np.float64)
    sq = 10 * np.log10((y ** 2).sum() / ((y - xh) ** 2).sum())
    assert st["sqnr_db"] == pytest.approx(sq, abs=0.05)                 # bf16 output rounding
    assert st["alpha"] == pytest.approx((y * xh).sum() / (y ** 2).sum(), rel=1e-3)
    assert st["cell_count"].sum() == x.size


def test_sqnr_direction_on_outlier_workload():
    # the pages' qualitative reversal across the rotation on an outlier-heavy tensor:
    # without RHT E2M1 >= E1M2; with RHT E1M2 > E2M1 (UFP4 page, RHT section; values unpinned)
    x = synth.outlier_activation(rows=128)
    mask = O.sign_mask_from_seed(synth.sign_seed(1))
    sq = {}
    for grid in (O.GRID_E2M1, O.GRID_E1M2):
        for rht in (0, 1):
            raw = O.quantize(O.OracleConfig(grid=grid, rht=rht, sign_mask=mask), x, stats=True)["stats_raw"]
            sq[grid, rht] = O.finalize_stats(raw)["sqnr_db"]
    assert sq[O.GRID_E2M1, 0] >= sq[O.GRID_E1M2, 0]
    assert sq[O.GRID_E1M2, 1] > sq[O.GRID_E2M1, 1]
    assert sq[O.GRID_E1M2, 1] > sq[O.GRID_E1M2, 0] and sq[O.GRID_E2M1, 1] < sq[O.GRID_E2M1, 0]


def test_sr_index_is_logical_row_major():
    # R12: element (m, n) of a row-orientation tensor uses idx = m * cols + n, so quantizing a
    # row range with row0 gives the same codes as the same rows inside the full tensor
    x = synth.small(81, 32, 64, "normal")
    cfg = O.OracleConfig(grid=O.GRID_E1M2, round=O.ROUND_SR, sign_mask=0x2222, sr_seed=99)
    full = O.quantize(cfg, x)
    part = O.quantize(cfg, np.ascontiguousarray(x[10:20]), row0=10)
    np.testing.assert_array_equal(full["codes"][10:20], part["codes"])
    other = O.quantize(cfg, np.ascontiguousarray(x[10:20]), row0=0)
    assert not np.array_equal(other["codes"], part["codes"])


# ------------------------------------------------------------------ pins from decoded outputs

_E4M3_TABLE = None


def _e4m3_table():
    global _E4M3_TABLE
    if _E4M3_TABLE is None:
        _E4M3_TABLE = np.array([O.e4m3_decode(b) for b in range(128)], np.float32)
    return _E4M3_TABLE


def _decoded_blocks(cfg, r, x):
    """From the input and the oracle's codes and scales alone: per element y (rotated, FP32),
    v = y / s (FP32 IEEE division, the scaled value), the decoded value in scaled units, its
    magnitude cell, and xhat = value * s (FP32); per block the IF4 INT4 flag."""
    rows, cols = x.shape
    bs = 32 if cfg.scale == O.SCALE_UE8M0_1x32 else 16
    xf = synth.bf16_bits_to_f32(x).reshape(-1, 16)
    y = np.stack([O.rht16(b, cfg.sign_mask) if cfg.rht else b for b in xf]).reshape(rows, cols)
    y = y.astype(np.float32)
    sc = r["scales"]
    flag = np.zeros(sc.shape, bool)
    if cfg.scale == O.SCALE_FP32_1x16:
        s = sc.astype(np.float32)
    elif cfg.scale == O.SCALE_E4M3_1x16:
        s = _e4m3_table()[sc & 0x7F] * np.float32(r["tensor_scale"])
        flag = (sc >> 7).astype(bool) if cfg.grid == O.GRID_IF4 else flag
    else:
        s = np.ldexp(np.float32(1), sc.astype(np.int32) - 127).astype(np.float32)
    s_el = np.repeat(s, bs, axis=1)
    int_el = np.repeat(flag, bs, axis=1)
    nib = _nib(r["codes"])
    fp_grid = O.GRID_E2M1 if cfg.grid == O.GRID_IF4 else cfg.grid
    k = _value_of(O.GRID_INT4, nib).astype(np.float32)
    if cfg.grid == O.GRID_INT4:
        val, cell = k, np.abs(k).astype(int)
    else:
        val, cell = _value_of(fp_grid, nib).astype(np.float32), (nib & 7).astype(int)
    val = np.where(int_el, k * np.float32(6 / 7), val).astype(np.float32)
    cell = np.where(int_el, np.abs(k).astype(int), cell)
    zero = s_el == 0
    with np.errstate(divide="ignore", invalid="ignore"):
        v = np.where(zero, np.float32(0), y / np.where(zero, np.float32(1), s_el)).astype(np.float32)
    xhat = np.where(zero, np.float32(0), val * s_el).astype(np.float32)
    return y, v, val, cell, xhat, flag


@pytest.mark.parametrize("name,cfg", [
    ("e1m2_fp32_rht", O.OracleConfig(grid=O.GRID_E1M2, sign_mask=0x1111)),
    ("int4_fp32_sr", O.OracleConfig(grid=O.GRID_INT4, round=O.ROUND_SR, sign_mask=0x0FF0, sr_seed=17)),
    ("e2m1max3_fp32", O.OracleConfig(grid=O.GRID_E2M1_MAX3, rht=0)),
    ("nvint4", O.OracleConfig(grid=O.GRID_INT4, scale=O.SCALE_E4M3_1x16, sign_mask=0x3003)),
    ("if4", O.OracleConfig(grid=O.GRID_IF4, scale=O.SCALE_E4M3_1x16, sign_mask=0x5A5A)),
    ("mxfp4", O.OracleConfig(grid=O.GRID_E2M1, scale=O.SCALE_UE8M0_1x32, sign_mask=0x0001)),
])
def test_stats_are_the_sums_over_decoded_codes(name, cfg):
    # UFP4-A (RHT and compounding sections) defines SQNR from sum y^2 / sum (y - xhat)^2 and the
    # attenuation from <xhat, y> / |y|^2; the E2M1 section the per-cell signed error in scaled
    # units; IF4 6.2 the share of blocks that keep FP4. Every raw sum is recomputed here from
    # the codes and scales, so a sum over the wrong operand or cell cannot pass.
    x = synth.small(97, 48, 256, "t4")
    r = O.quantize(cfg, x, stats=True)
    raw = r["stats_raw"]
    y, v, val, cell, xhat, flag = _decoded_blocks(cfg, r, x)
    y64, xh64 = y.astype(np.float64), xhat.astype(np.float64)
    np.testing.assert_allclose(raw[O.ST_SUM_Y2], (y64 ** 2).sum(), rtol=1e-12)
    np.testing.assert_allclose(raw[O.ST_SUM_ERR2], ((y64 - xh64) ** 2).sum(), rtol=1e-12)
    np.testing.assert_allclose(raw[O.ST_SUM_YXHAT], (y64 * xh64).sum(), rtol=1e-12)
    assert raw[O.ST_N] == x.size
    err = np.abs(val.astype(np.float64)) - np.abs(v.astype(np.float64))
    for c in range(8):
        assert raw[O.ST_CELL_N + c] == (cell == c).sum(), c
        np.testing.assert_allclose(raw[O.ST_CELL_ERR + c], err[cell == c].sum(), rtol=1e-9, atol=1e-9)
    assert raw[O.ST_BLOCKS] == r["scales"].size
    if cfg.grid == O.GRID_IF4:
        assert 0 < flag.sum() < flag.size
        assert raw[O.ST_IF4_FP4] == (~flag).sum()


def test_if4_picks_the_smaller_squared_error_brute_force():
    # IF4 sections 3.1 / 3.1.1: each block keeps the candidate with the smaller mean squared
    # error; INT4 only when strictly smaller (R11). Both candidates are formed here from v by
    # brute force: E2M1 by the exponent/step rule, INT4 as round-half-even(v * RN(7/6)) clamped to
    # 7 and valued k * RN(6/7); errors in FP64.
    cfg = O.OracleConfig(grid=O.GRID_IF4, scale=O.SCALE_E4M3_1x16, sign_mask=0x6C6C)
    checked = separated = 0
    for seed, kind in [(101, "uniform"), (102, "normal"), (103, "laplace"), (104, "t4")]:
        x = synth.small(seed, 128, 256, kind)
        r = O.quantize(cfg, x)
        _, v, _, _, _, flag = _decoded_blocks(cfg, r, x)
        v = v.reshape(-1, 16)
        fp = np.copysign(_e2m1_by_exponent(np.abs(v.astype(np.float64))), v)
        w = (v * np.float32(7 / 6)).astype(np.float32)
        k = np.clip(np.rint(w), -7, 7).astype(np.float32)
        it = (k * np.float32(6 / 7)).astype(np.float64)
        sse_fp = ((fp - v) ** 2).sum(-1)
        sse_int = ((it - v) ** 2).sum(-1)
        decided = np.abs(sse_int - sse_fp) > 1e-4 * np.maximum(sse_fp, 1e-30)
        want = sse_int < sse_fp
        got = flag.reshape(-1)
        np.testing.assert_array_equal(got[decided], want[decided])
        checked += decided.sum()
        # and each block carries the codes of the candidate it chose
        nib = _nib(r["codes"]).reshape(-1, 16)
        k_codes = (k.astype(np.int64) & 0xF).astype(np.uint8)
        np.testing.assert_array_equal(nib[got], k_codes[got])
        fp_vals = np.array([O.decode_nibble(O.GRID_E2M1, c) for c in range(16)])[nib[~got]]
        np.testing.assert_array_equal(np.abs(fp_vals), np.abs(fp[~got]))
        # blocks where the absolute error would choose the other way
        l1 = np.abs(it - v).sum(-1) < np.abs(fp - v).sum(-1)
        separated += (decided & (l1 != want)).sum()
    assert checked > 1500 and separated > 0
    # an exact tie: scaled values in {0, +-6} lie on both candidates (7 * RN(6/7) rounds to 6),
    # both errors are 0, and the block keeps FP4
    tie = np.array([6, 0, -6, 0] * 4, np.float32)
    assert np.float32(7) * np.float32(6 / 7) == np.float32(6)
    r = O.quantize(O.OracleConfig(grid=O.GRID_IF4, scale=O.SCALE_E4M3_1x16, rht=0),
                   synth.to_bf16_bits(tie[None]), tensor_scale=np.float32(1 / 64))
    # Delta = 6 / (6/64) = 64 = 2^6: E4M3 exponent field 6 + 7 = 13, mantissa 0 -> 0x68; bit 7
    # clear: FP4 kept
    assert r["scales"][0, 0] == 0x68


def test_sr_rounds_each_element_with_its_own_draw():
    # R12: element (m, n) draws u = sr_bits(seed, stream, m * cols + n). With every element half
    # way between two E1M2 points (v = 1.25, s = 1) it rounds up to 1.5 exactly when
    # u * 2^-16 < 1/2; the block's first element (3.5) sets s and is a grid point.
    rows, cols, row0 = 6, 64, 5
    row = np.full(cols, 1.25, np.float32)
    row[::16] = 3.5
    x = synth.to_bf16_bits(np.tile(row, (rows, 1)))
    for stream in (0, 1):
        cfg = O.OracleConfig(grid=O.GRID_E1M2, round=O.ROUND_SR, rht=0, sr_seed=1234, sr_stream=stream)
        nib = _nib(O.quantize(cfg, x, row0=row0)["codes"])
        want = np.empty((rows, cols), np.uint8)
        for m in range(rows):
            for n in range(cols):
                u = O.sr_bits(1234, stream, (row0 + m) * cols + n)
                want[m, n] = 7 if n % 16 == 0 else (3 if u < 2 ** 15 else 2)
        np.testing.assert_array_equal(nib, want)
        assert 0.3 < (want == 3).mean() < 0.7


def test_sign_mask_is_the_low_bits_of_the_published_outputs():
    # R1: the sign mask of a seed is the low 16 bits of SplitMix64's first output from that
    # state; from states 0 and gamma these are the first two published outputs
    outs = [int(ln[0], 16) for ln in _golden_lines("splitmix64.txt")]
    assert O.sign_mask_from_seed(0) == outs[0] & 0xFFFF
    assert O.sign_mask_from_seed(0x9E3779B97F4A7C15) == outs[1] & 0xFFFF


def test_nv_block_below_the_e4m3_range_encodes_zero():
    # R8: a block whose Delta = amax_b / (alpha * 6) rounds to E4M3 zero (below 2^-10, half the
    # smallest subnormal) has s = 0 and encodes as zeros, whatever its signs
    big = np.full(16, 448.0 * 6, np.float32)              # alpha = A / (6 * 448) = 1
    tiny = np.array([1e-4, -2e-4, 3e-4, -1e-4] * 4, np.float32)
    x = synth.to_bf16_bits(np.stack([big, tiny]))
    r = O.quantize(O.OracleConfig(grid=O.GRID_E2M1, scale=O.SCALE_E4M3_1x16, rht=0), x, dequant=True)
    assert r["tensor_scale"] == 1.0 and r["scales"][0, 0] == 0x7E
    assert r["scales"][1, 0] == 0
    assert np.all(r["codes"][1] == 0) and np.all(r["dequant"][1] == 0)


def test_row_pitch_is_layout_only():
    # a row pitch larger than the row (ld > cols) changes where rows start, not what is
    # quantized: a view into a wider array gives the outputs of its contiguous copy, with the
    # padding columns (filled with large values) never read
    wide = synth.small(111, 40, 320, "laplace", 2.0)
    wide[:, 256:] = synth.to_bf16_bits(np.full((40, 64), 1e4, np.float32))
    view = wide[:, :256]
    dense = np.ascontiguousarray(view)
    assert view.strides[0] == 640 and dense.strides[0] == 512
    for cfg in (O.OracleConfig(grid=O.GRID_E1M2, sign_mask=0x4321),
                O.OracleConfig(grid=O.GRID_E2M1, scale=O.SCALE_E4M3_1x16, sign_mask=0x4321),
                O.OracleConfig(grid=O.GRID_E2M1, scale=O.SCALE_UE8M0_1x32, sign_mask=0x4321)):
        a, b = O.quantize(cfg, view, dequant=True), O.quantize(cfg, dense, dequant=True)
        for key in ("codes", "scales", "dequant"):
            np.testing.assert_array_equal(a[key], b[key])
        assert a["tensor_scale"] == b["tensor_scale"]
        assert O.tensor_amax(cfg, view) == O.tensor_amax(cfg, dense)
    for ya, yb in zip(O.rht16_rows(view, 0x4321), O.rht16_rows(dense, 0x4321)):
        np.testing.assert_array_equal(ya, yb)


def test_format_error_ranking_on_laplace():
    # IF4 page, section 2.2 table: MXFP4 > NVFP4 > NVINT4 > IF4 in quantization MSE (values
    # printed without their data, so only the order is pinned), and IF4 keeps FP4 on part of
    # the blocks (section 6.2); on a Laplace sample with the rotation
    x = synth.laplace_format_tensor(rows=512)
    mask = O.sign_mask_from_seed(synth.sign_seed(4))
    nmse = {}
    for name, grid, scale in (("MXFP4", O.GRID_E2M1, O.SCALE_UE8M0_1x32),
                              ("NVFP4", O.GRID_E2M1, O.SCALE_E4M3_1x16),
                              ("NVINT4", O.GRID_INT4, O.SCALE_E4M3_1x16),
                              ("IF4", O.GRID_IF4, O.SCALE_E4M3_1x16)):
        st = O.finalize_stats(O.quantize(O.OracleConfig(grid=grid, scale=scale, sign_mask=mask), x,
                                         stats=True)["stats_raw"])
        nmse[name] = st["nmse"]
        if grid == O.GRID_IF4:
            assert 0.1 < st["if4_fp4_fraction"] < 0.9
    assert nmse["MXFP4"] > nmse["NVFP4"] > nmse["NVINT4"] > nmse["IF4"]
