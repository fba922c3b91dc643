"""Pins of the oracle's power-of-two scale mode (the scale factors a tensor
core can apply itself; not the pages' S = amax/448, which stays the default).

Definition checked: S = 2^e with e the smallest integer such that the tile's
amax <= 448 * 2^e (held at 2^-127 or above; S = 0 for an all-zero tile), and
codes = E4M3 round-to-nearest-even of x / S, which is exact for a power of
two.  The checks use properties of that definition, numpy's exact frexp /
ldexp, and an independent library cast (PyTorch float8_e4m3fn)."""
import numpy as np
import torch

from moe_synth import gen_gemm_a, normal_bf16

POW2 = 1


def _tiles(x, rows, groups):
    return np.abs(x.float().numpy().reshape(rows, groups, 128)).max(axis=2).astype(np.float64)


def test_pow2_scale_is_the_smallest_power_of_two_that_fits(oracle_lib):
    x = gen_gemm_a(64, 1024, 0)
    q, s = oracle_lib.quant_1x128(x, POW2)
    amax = _tiles(x, 64, 8)
    s = s.astype(np.float64)
    mant, _ = np.frexp(s)
    assert np.all(mant == 0.5)                  # exact powers of two
    assert np.all(amax <= 448.0 * s)            # the tile fits ...
    assert np.all(amax > 448.0 * (s / 2))       # ... and would not at half the scale
    # relation to the pages' scale: amax/448 <= S < 2 * amax/448
    assert np.all(s >= amax / 448.0) and np.all(s < 2 * amax / 448.0)


def test_pow2_codes_match_library_cast_of_the_exact_quotient(oracle_lib):
    x = gen_gemm_a(64, 1024, 1)
    q, s = oracle_lib.quant_1x128(x, POW2)
    quot = x.double().reshape(64, 8, 128) / torch.from_numpy(s.astype(np.float64)).reshape(64, 8, 1)
    # the quotient by a power of two is exact, so its float32 form loses nothing
    assert torch.equal(quot.float().double(), quot)
    lib = quot.float().clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8).reshape(64, 1024).numpy()
    assert np.array_equal(q, lib)


def test_pow2_boundaries(oracle_lib):
    # amax exactly 448 * 2^j fits at 2^j; one bf16 step above needs 2^(j+1);
    # amax 224 = 448 / 2 fits at 1/2
    for amax, want in [(448.0, 1.0), (450.0, 2.0), (224.0, 0.5), (1.0, 2.0 ** -8), (896.0, 2.0)]:
        x = torch.zeros(1, 128, dtype=torch.bfloat16)
        x[0, 5] = amax
        x[0, 9] = -amax / 3
        q, s = oracle_lib.quant_1x128(x, POW2)
        assert float(s[0, 0]) == want, (amax, float(s[0, 0]))
    z = torch.zeros(2, 256, dtype=torch.bfloat16)
    q, s = oracle_lib.quant_1x128(z, POW2)
    assert not q.any() and not s.any()


def test_pow2_scaling_by_powers_of_two_shifts_the_scale_only(oracle_lib):
    x = normal_bf16((16, 512), 1.0, 5)
    q0, s0 = oracle_lib.quant_1x128(x, POW2)
    for j in (-7, 3):
        q1, s1 = oracle_lib.quant_1x128((x.float() * 2.0 ** j).bfloat16(), POW2)
        assert np.array_equal(q1, q0)
        assert np.array_equal(s1, s0 * np.float32(2.0 ** j))


def test_pow2_error_bound(oracle_lib):
    x = gen_gemm_a(128, 1024, 3)
    q, s = oracle_lib.quant_1x128(x, POW2)
    xd = oracle_lib.dequant(q, s, 1)
    xf = x.double().numpy()
    S = np.repeat(s.astype(np.float64), 128, axis=1)
    err = np.abs(xd - xf)
    normal = np.abs(xf) >= S * 2.0 ** -6
    assert np.all(err[normal] <= 2.0 ** -4 * np.abs(xf[normal]))
    assert np.all(err[~normal] <= 2.0 ** -10 * S[~normal])


def test_pow2_weight_blocks(oracle_lib):
    w = normal_bf16((256, 384), 0.02, 7)
    q, s = oracle_lib.quant_128x128(w, POW2)
    amax = np.abs(w.float().numpy().reshape(2, 128, 3, 128)).max(axis=(1, 3)).astype(np.float64)
    s = s.astype(np.float64)
    assert np.all(np.frexp(s)[0] == 0.5)
    assert np.all(amax <= 448.0 * s) and np.all(amax > 224.0 * s)
    quot = w.double().reshape(2, 128, 3, 128) / torch.from_numpy(s).reshape(2, 1, 3, 1)
    lib = quot.float().to(torch.float8_e4m3fn).view(torch.uint8).reshape(256, 384).numpy()
    assert np.array_equal(q, lib)


def test_pow2_f32_input(oracle_lib):
    rng = np.random.default_rng(11)
    h = (rng.standard_normal((8, 256)) * 3).astype(np.float32)
    q, s = oracle_lib.quant_1x128_f32(h, POW2)
    amax = np.abs(h.reshape(8, 2, 128)).max(axis=2).astype(np.float64)
    s = s.astype(np.float64)
    assert np.all(amax <= 448.0 * s) and np.all(amax > 224.0 * s)
    quot = torch.from_numpy(h.astype(np.float64).reshape(8, 2, 128) / s.reshape(8, 2, 1))
    lib = quot.float().to(torch.float8_e4m3fn).view(torch.uint8).reshape(8, 256).numpy()
    assert np.array_equal(q, lib)
