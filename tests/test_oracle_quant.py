"""Pins of the oracle's fine-grained quantizers.

What the pages fix ("DeepSeek-V3 Technischer Bericht", Kernideen FP8 bullet;
"DeepSeek-V3 技術報告書" formula paragraph; slideify "FP8 Quantization Logic"):
one scale per 1x128 activation tile and per 128x128 weight block,
S = max|X| / 448, X_FP8 = clip(round(X / S), -448, 448).  The checks below are
properties any implementation of that definition has, plus an independent
library cast (PyTorch float8_e4m3fn) applied to the same quotients.
"""
import numpy as np
import pytest
import torch

from moe_synth import gen_gemm_a, normal_bf16


def _x_with_outliers(rows, cols, seed):
    return gen_gemm_a(rows, cols, seed)


def _deq(oracle_lib, q, s, br):
    return oracle_lib.dequant(q, s, br)


def test_1x128_scale_is_tile_amax_over_448(oracle_lib):
    x = _x_with_outliers(64, 1024, 0)
    q, s = oracle_lib.quant_1x128(x)
    xf = x.float().numpy().reshape(64, 8, 128)
    amax = np.abs(xf).max(axis=2).astype(np.float32)
    assert np.array_equal(s, amax / np.float32(448.0))


def test_1x128_codes_match_library_cast(oracle_lib):
    x = _x_with_outliers(64, 1024, 1)
    q, s = oracle_lib.quant_1x128(x)
    quot = (x.float().reshape(64, 8, 128) / torch.from_numpy(s).reshape(64, 8, 1)).reshape(64, 1024)
    assert torch.isfinite(quot).all()
    lib = quot.clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(q, lib)


def test_1x128_amax_element_maps_to_448(oracle_lib):
    x = _x_with_outliers(32, 512, 2)
    q, s = oracle_lib.quant_1x128(x)
    xf = x.float().numpy().reshape(32, 4, 128)
    arg = np.abs(xf).argmax(axis=2)
    qq = q.reshape(32, 4, 128)
    for r in range(32):
        for g in range(4):
            c = qq[r, g, arg[r, g]]
            assert c == (0x7E if xf[r, g, arg[r, g]] > 0 else 0xFE)


def test_1x128_error_bound(oracle_lib):
    x = _x_with_outliers(128, 1024, 3)
    q, s = oracle_lib.quant_1x128(x)
    xd = _deq(oracle_lib, q, s, 1)
    xf = x.double().numpy()
    S = np.repeat(s.astype(np.float64), 128, axis=1)
    err = np.abs(xd - xf)
    normal = np.abs(xf) / S >= 2.0 ** -6
    # normal range: 3 mantissa bits, RNE -> relative error <= 2^-4
    assert np.all(err[normal] <= 2.0 ** -4 * np.abs(xf[normal]) * (1 + 1e-6))
    # subnormal range: absolute error <= half a subnormal step times S
    assert np.all(err[~normal] <= 2.0 ** -10 * S[~normal] * (1 + 1e-6))


def test_1x128_power_of_two_invariance(oracle_lib):
    x = normal_bf16((16, 512), 1.0, 4)
    q, s = oracle_lib.quant_1x128(x)
    for j in (-3, 5):
        q2, s2 = oracle_lib.quant_1x128((x.float() * 2.0 ** j).to(torch.bfloat16))
        assert np.array_equal(q, q2)
        assert np.array_equal(s2, s * np.float32(2.0 ** j))


def test_1x128_zero_tile(oracle_lib):
    x = normal_bf16((4, 256), 1.0, 5)
    x[1, 128:] = 0
    q, s = oracle_lib.quant_1x128(x)
    assert s[1, 1] == 0.0 and np.all(q[1, 128:] == 0)


def test_1x128_f32_matches_bf16_path_on_bf16_values(oracle_lib):
    x = _x_with_outliers(16, 512, 6)
    q1, s1 = oracle_lib.quant_1x128(x)
    q2, s2 = oracle_lib.quant_1x128_f32(x.float().numpy())
    assert np.array_equal(q1, q2) and np.array_equal(s1, s2)


def test_128x128_scale_and_codes(oracle_lib):
    w = normal_bf16((256, 384), 0.02, 7)
    w[5, 7] = 0.9  # an outlier in block (0, 0)
    q, s = oracle_lib.quant_128x128(w)
    wf = w.float().numpy()
    amax = np.abs(wf.reshape(2, 128, 3, 128)).max(axis=(1, 3)).astype(np.float32)
    assert np.array_equal(s, amax / np.float32(448.0))
    quot = torch.from_numpy(wf.reshape(2, 128, 3, 128) / s[:, None, :, None]).reshape(256, 384)
    lib = quot.clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(q, lib)
    assert q[5, 7] == 0x7E
    wd = _deq(oracle_lib, q, s, 128)
    Sx = np.repeat(np.repeat(s.astype(np.float64), 128, 0), 128, 1)
    normal = np.abs(wf) / Sx >= 2.0 ** -6
    err = np.abs(wd - wf)
    assert np.all(err[normal] <= 2.0 ** -4 * np.abs(wf[normal]) * (1 + 1e-6))
    assert np.all(err[~normal] <= 2.0 ** -10 * Sx[~normal] * (1 + 1e-6))
