"""Pins of the oracle's E4M3 codec.

The pages fix E4M3 for all tensors and the clip bound 448 ("DeepSeek-V3
Technischer Bericht", Kernideen FP8 bullet; "DeepSeek-V3 技術報告書" formula
paragraph).  The codec is pinned against PyTorch's float8_e4m3fn dtype (an
independent library implementation of the OCP E4M3FN format) and against
properties any correct round-to-nearest-even, saturating cast must have.
"""
import math

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.filterwarnings("ignore")


def test_decode_matches_library_for_all_codes(oracle_lib):
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    lib_vals = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = oracle_lib.e4m3_decode_table()
    for c in range(256):
        if math.isnan(lib_vals[c]):
            assert math.isnan(ours[c]), c
            assert c in (0x7F, 0xFF)
        else:
            assert ours[c] == lib_vals[c], (c, ours[c], lib_vals[c])


def test_decode_structure(oracle_lib):
    t = oracle_lib.e4m3_decode_table()
    assert t[0x7E] == 448.0 and t[0xFE] == -448.0          # clip bound of the pages
    assert t[0x01] == 2.0 ** -9                             # smallest subnormal
    assert t[0x08] == 2.0 ** -6                             # smallest normal
    assert t[0x00] == 0.0 and math.copysign(1, t[0x80]) < 0  # signed zeros
    pos = t[:0x7F]
    assert np.all(np.diff(pos) > 0)                         # strictly increasing
    for c in range(0x7F):
        assert t[c | 0x80] == -t[c]


def _finite_codes():
    return [c for c in range(0x7F)]


def test_encode_roundtrip_every_code(oracle_lib):
    t = oracle_lib.e4m3_decode_table()
    for c in _finite_codes():
        assert oracle_lib.e4m3_encode(t[c]) == c
        assert oracle_lib.e4m3_encode(-t[c]) == (c | 0x80)


def test_encode_midpoints_round_to_even(oracle_lib):
    t = oracle_lib.e4m3_decode_table()
    for c in range(0x7E):
        lo, hi = t[c], t[c + 1]
        mid = (lo + hi) / 2.0
        assert float(np.float32(mid)) == mid  # representable in fp32
        even = c if (c & 1) == 0 else c + 1
        assert oracle_lib.e4m3_encode(mid) == even, (c, mid)
        below = float(np.nextafter(np.float32(mid), np.float32(0)))
        above = float(np.nextafter(np.float32(mid), np.float32(1e9)))
        assert oracle_lib.e4m3_encode(below) == c
        assert oracle_lib.e4m3_encode(above) == c + 1


def test_encode_saturates_and_special_values(oracle_lib):
    enc = oracle_lib.e4m3_encode
    for v in (448.0, 449.0, 463.9, 464.0, 480.0, 1e6, 3.0e38):
        assert enc(v) == 0x7E and enc(-v) == 0xFE
    assert enc(0.0) == 0x00 and enc(-0.0) == 0x80
    assert enc(2.0 ** -9) == 0x01
    assert enc(2.0 ** -10) == 0x00          # half of the smallest subnormal: tie to even (0)
    assert enc(3 * 2.0 ** -10) == 0x02      # tie between 1 and 2 subnormal steps -> 2
    assert enc(15 * 2.0 ** -10) == 0x08     # tie between 7/8 subnormal and 2^-6 -> even (0x08)


def test_encode_matches_library_cast_in_range(oracle_lib):
    rng = np.random.default_rng(0)
    vals = np.concatenate([
        rng.standard_normal(20000) * 50.0,
        rng.standard_normal(20000) * 1e-2,
        rng.uniform(-448, 448, 20000),
        (rng.standard_normal(5000) * 1e-3),
    ]).astype(np.float32)
    lib_codes = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = np.array([oracle_lib.e4m3_encode(float(v)) for v in vals], dtype=np.uint8)
    assert np.array_equal(ours, lib_codes)
