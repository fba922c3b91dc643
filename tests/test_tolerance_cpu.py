"""CPU checks of the near-tie allowance the parity tests add to the max bound
(``_moe_util.near_tie_steps``): it flags exactly the quotients that sit near
a rounding midpoint of the E4M3 grid, with the size of the code step, and it
covers what a last-bit difference of an FP32 intermediate does downstream:
two copies of a matrix one ulp apart, each quantized 1x128 by the oracle and
multiplied into a GEMM, differ by no more than the allowance of either."""
import numpy as np
import pytest

from _moe_util import TIE_BAND, near_tie_steps, tiles_1x128


@pytest.fixture(scope="module")
def dec(oracle_lib):
    return oracle_lib.e4m3_decode_table()


def test_midpoints_and_grid_points(dec):
    # 1.0 and 1.125 are neighbours (3 mantissa bits): their midpoint is a tie
    v = np.array([1.0625, -1.0625, 1.0, 1.0625 * (1 + 2e-4), 300.0, 304.0, 448.0, 0.0])
    got = near_tie_steps(v, np.ones_like(v), dec)
    # 300 lies between 288 and 320 (midpoint 304)
    assert got.tolist() == [0.125, 0.125, 0.0, 0.0, 0.0, 32.0, 0.0, 0.0]
    # a wider band takes the value 2e-4 off the midpoint in
    assert near_tie_steps(v[3:4], np.ones(1), dec, band=1e-3)[0] == 0.125


def test_scale_and_absolute_band_below_one(dec):
    # the step is in units of the scale
    assert near_tie_steps(np.array([2.125]), np.array([2.0]), dec)[0] == 0.25
    # subnormal codes: 2^-9 and 2^-8 have the midpoint 1.5 * 2^-9; below a
    # quotient of 1 the band is absolute
    m = 1.5 * 2.0 ** -9
    assert near_tie_steps(np.array([m + 5e-5]), np.ones(1), dec)[0] == 2.0 ** -9
    assert near_tie_steps(np.array([m + 5e-4]), np.ones(1), dec)[0] == 0.0
    # a zero scale (an all-zero tile) has no ties
    assert near_tie_steps(np.array([0.0]), np.zeros(1), dec)[0] == 0.0


def test_allowance_covers_last_bit_differences(oracle_lib, dec):
    rng = np.random.default_rng(0)
    rows, K, N = 64, 512, 96
    a = (rng.standard_normal((rows, K)) * rng.uniform(0.1, 10, size=(rows, 1))).astype(np.float32)
    # plant exact midpoints: v = mid * S with S = amax / 448 of the tile
    a[:, :128] = 0.0
    a[:, 0] = 448.0
    a[:, 1:9] = np.float32(1.0625)
    b = a.copy()
    # the other side's rounding: one ulp up or down, everywhere
    b = np.nextafter(b, np.where(rng.random(b.shape) < 0.5, np.inf, -np.inf).astype(np.float32)).astype(np.float32)
    b[:, 0] = 448.0  # the same tile scale on both sides
    w = rng.standard_normal((N, K))
    qa, sa = oracle_lib.quant_1x128_f32(a)
    qb, sb = oracle_lib.quant_1x128_f32(b)
    ya = (dec[qa] * tiles_1x128(sa)) @ w.T
    yb = (dec[qb] * tiles_1x128(sb)) @ w.T
    allow = near_tie_steps(a.astype(np.float64), tiles_1x128(sa), dec) @ np.abs(w.T)
    assert (dec[qa] != dec[qb]).any(), "no code moved: the check would be vacuous"
    # FP32 rounding of the scales apart, the change is within the allowance
    assert np.all(np.abs(ya - yb) <= allow + 1e-5 * np.abs(ya).max())
    # and the allowance is not everything: off the ties it is zero
    steps = near_tie_steps(a.astype(np.float64), tiles_1x128(sa), dec)
    assert (steps > 0).mean() < 0.05
    assert TIE_BAND == 1e-4
