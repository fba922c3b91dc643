"""Pins of the oracle (and of the package's defaults) to the numbers the pages
print, stored with their citations in ``tests/golden/page_constants.txt``.

Each check is a behaviour that a wrong constant would break: a clip bound
other than 448 changes the largest code, a tile other than 1x128 or a block
other than 128x128 lets a change in one tile move another tile's scale, a
promotion interval other than 128 applies a K-block's scale to the wrong
columns, and a bias step other than gamma moves the bias by another amount.
"""
import inspect
import os

import numpy as np
import pytest

import moe_synth
from moe_synth import normal_bf16

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "page_constants.txt")


def _load():
    out = {}
    with open(GOLDEN, encoding="utf-8") as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            lhs, cite = line.split("|", 1)
            name, value = (t.strip() for t in lhs.split("=", 1))
            assert cite.strip(), f"{name} has no citation"
            out[name] = float(value)
    return out


G = _load()


def test_fixture_lists_every_constant():
    assert set(G) == {"fp8_clip", "scale_divisor", "act_tile_rows", "act_tile_cols", "weight_block_rows",
                      "weight_block_cols", "promotion_interval", "gamma", "n_routed", "n_shared", "top_k"}


def test_clip_bound_is_the_largest_finite_code(oracle_lib):
    table = oracle_lib.e4m3_decode_table()
    finite = table[np.isfinite(table)]
    assert finite.max() == G["fp8_clip"] and finite.min() == -G["fp8_clip"]
    assert oracle_lib.e4m3_decode(oracle_lib.e4m3_encode(1e30)) == G["fp8_clip"]
    assert oracle_lib.e4m3_decode(oracle_lib.e4m3_encode(-1e30)) == -G["fp8_clip"]


def test_scale_divides_the_tile_amax_by_the_printed_divisor(oracle_lib):
    x = normal_bf16((4, 256), std=1.0, seed=11)
    q, s = oracle_lib.quant_1x128(x)
    amax = np.abs(x.float().numpy()).reshape(4, 2, 128).max(axis=2).astype(np.float32)
    assert np.array_equal(s, amax / np.float32(G["scale_divisor"]))
    # the amax element lands on the clip bound
    dec = oracle_lib.e4m3_decode_table()[q].reshape(4, 2, 128)
    assert np.array_equal(np.abs(dec).max(axis=2), np.full((4, 2), G["fp8_clip"]))


def test_activation_tile_is_one_row_by_128_columns(oracle_lib):
    rows, cols = 3, 384
    tr, tc = int(G["act_tile_rows"]), int(G["act_tile_cols"])
    x = normal_bf16((rows, cols), std=1.0, seed=12)
    q0, s0 = oracle_lib.quant_1x128(x)
    assert s0.shape == (rows // tr, cols // tc)
    y = x.clone()
    y[1, 200] = 64.0  # a new amax inside tile (row 1, columns 128..255)
    q1, s1 = oracle_lib.quant_1x128(y)
    changed = s1 != s0
    assert changed[1, 1] and changed.sum() == 1
    diff = np.argwhere(q1 != q0)
    assert diff.size and (diff[:, 0] == 1).all() and (diff[:, 1] >= tc).all() and (diff[:, 1] < 2 * tc).all()


def test_weight_block_is_128_by_128(oracle_lib):
    n, k = 256, 384
    br, bc = int(G["weight_block_rows"]), int(G["weight_block_cols"])
    w = normal_bf16((n, k), seed=13, std=0.02)
    q0, s0 = oracle_lib.quant_128x128(w)
    assert s0.shape == (n // br, k // bc)
    v = w.clone()
    v[130, 300] = 8.0  # inside block (1, 2)
    q1, s1 = oracle_lib.quant_128x128(v)
    changed = s1 != s0
    assert changed[1, 2] and changed.sum() == 1
    diff = np.argwhere(q1 != q0)
    assert diff.size
    assert ((diff[:, 0] >= br) & (diff[:, 0] < 2 * br) & (diff[:, 1] >= 2 * bc)).all()


def test_each_k_block_scale_covers_exactly_the_promotion_interval(oracle_lib):
    nc = int(G["promotion_interval"])
    M, N, K = 8, 256, 3 * nc
    qa, sa = oracle_lib.quant_1x128(normal_bf16((M, K), std=1.0, seed=14))
    qb, sb = oracle_lib.quant_128x128(normal_bf16((N, K), seed=15, std=0.02))
    full = oracle_lib.blockscaled_gemm(qa, sa, qb, sb)
    for kb in range(K // nc):
        # zero the scale of K-block kb ...
        sa_z = sa.copy()
        sa_z[:, kb] = 0.0
        # ... or zero its codes: both must drop the same columns of K
        qa_z = qa.copy()
        qa_z[:, kb * nc:(kb + 1) * nc] = 0
        a = oracle_lib.blockscaled_gemm(qa, sa_z, qb, sb)
        b = oracle_lib.blockscaled_gemm(qa_z, sa, qb, sb)
        assert np.array_equal(a, b)
        assert not np.allclose(a, full)
    # the K-block partials add up to the whole product
    parts = []
    for kb in range(K // nc):
        keep = np.zeros_like(sa)
        keep[:, kb] = sa[:, kb]
        parts.append(oracle_lib.blockscaled_gemm(qa, keep, qb, sb))
    np.testing.assert_allclose(sum(parts), full, rtol=1e-12, atol=0)
    # a weight block row of scales covers 128 output columns
    sb_z = sb.copy()
    sb_z[1, :] = 0.0
    c = oracle_lib.blockscaled_gemm(qa, sa, qb, sb_z)
    assert np.array_equal(c[:, :128], full[:, :128]) and not c[:, 128:].any()


def test_bias_moves_by_gamma(oracle_lib):
    g = np.float32(G["gamma"])
    Nr, Kr, T = 4, 2, 8  # mean load T*Kr/Nr = 4
    counts = np.array([6, 2, 4, 4], np.int32)
    b = oracle_lib.bias_update(np.zeros(Nr, np.float32), counts, Nr, T * Kr, gamma=float(g))
    assert b.tolist() == [-g, g, 0.0, 0.0]


def test_package_and_oracle_default_to_the_printed_gamma(oracle_lib):
    from sparse_moe_layer_expert_b200 import _binding
    from sparse_moe_layer_expert_b200.layer import MoeLayer
    assert inspect.signature(oracle_lib.bias_update).parameters["gamma"].default == G["gamma"]
    assert inspect.signature(_binding.moe_bias_update).parameters["gamma"].default == G["gamma"]
    assert inspect.signature(MoeLayer.bias_update).parameters["gamma"].default == G["gamma"]


@pytest.mark.parametrize("name", ["decode", "prefill", "skewed"])
def test_v3_workloads_use_the_printed_expert_counts(name):
    c = moe_synth.CONFIGS[name]
    assert c["Nr"] == G["n_routed"] and c["Ns"] == G["n_shared"] and c["Kr"] == G["top_k"]
