"""Pins of the oracle's expert FFN, layer combine and bias update.

"DeepSeek-V3 Technischer Bericht", Methode section 2:
h'_t = u_t + sum_{i<=N_s} FFN^(s)_i(u_t) + sum_{i<=N_r} g_{i,t} FFN^(r)_i(u_t),
and the per-step bias rule b_i -= gamma when expert i is overloaded, += gamma
when underloaded (gamma = 0.001).  The FFN is SwiGLU, W2(silu(W1 u) * W3 u),
with FP8 operands on both projections.

Pins: the FFN against library matmuls of dequantized operands; the layer
against the identity that makes routing irrelevant (all routed experts equal
=> output = u + FFN_shared(u) + FFN_routed(u) because the gates sum to one);
the bias update against its closed form.
"""
import numpy as np
import pytest
import torch

from moe_synth import TINY, gen_bias, gen_expert, gen_router, gen_x


def _quant_expert(oracle_lib, e, H, I, seed, mode=0):
    w13, w2 = gen_expert(e, H, I, seed)
    W13q, s13 = oracle_lib.quant_128x128(w13, mode)
    W2q, s2 = oracle_lib.quant_128x128(w2, mode)
    return W13q, s13, W2q, s2


# scale mode 0: S = amax/448 (the pages); 1: power-of-two scales
@pytest.mark.parametrize("mode", [0, 1])
def test_ffn_matches_dense_swiglu_of_dequantized(oracle_lib, mode):
    H, I = 512, 256
    cf = oracle_lib.cfg(H, I, 4, 2, scale_mode=mode)
    x = gen_x(24, H, 0)
    xq, xs = oracle_lib.quant_1x128(x, mode)
    W13q, s13, W2q, s2 = _quant_expert(oracle_lib, 0, H, I, 0, mode)
    y, h, hq, hs = oracle_lib.expert_ffn(cf, xq, xs, W13q, s13, W2q, s2, want_h=True)
    Xd = oracle_lib.dequant(xq, xs, 1)
    W13d = oracle_lib.dequant(W13q, s13, 128)
    GU = Xd @ W13d.T
    G = GU[:, :I].astype(np.float32).astype(np.float64)
    U = GU[:, I:].astype(np.float32).astype(np.float64)
    h_ref = (G / (1.0 + np.exp(-G)) * U).astype(np.float32)
    assert np.allclose(h, h_ref, rtol=2e-7, atol=0)
    hq_ref, hs_ref = oracle_lib.quant_1x128_f32(h_ref, mode)
    assert (hq == hq_ref).mean() > 0.9999
    W2d = oracle_lib.dequant(W2q, s2, 128)
    y_ref = oracle_lib.dequant(hq_ref, hs_ref, 1) @ W2d.T
    assert np.allclose(y, y_ref, rtol=0, atol=1e-6 * np.abs(y_ref).max())


@pytest.mark.parametrize("mode", [0, 1])
def test_layer_identity_all_routed_experts_equal(oracle_lib, mode):
    c = TINY
    H, I, Nr, Kr = c["H"], c["I"], c["Nr"], c["Kr"]
    cf = oracle_lib.cfg(H, I, Nr, Kr, scale_mode=mode)
    x = gen_x(32, H, 1)
    Wr = gen_router(Nr, H, 1)
    b = gen_bias(Nr, 1)
    shared = _quant_expert(oracle_lib, Nr, H, I, 1, mode)
    same = _quant_expert(oracle_lib, 0, H, I, 1, mode)
    res = oracle_lib.forward(cf, x, Wr, b, [same] * Nr + [shared])
    xq, xs = oracle_lib.quant_1x128(x, mode)
    y_sh = oracle_lib.expert_ffn(cf, xq, xs, *shared)
    y_w = oracle_lib.expert_ffn(cf, xq, xs, *same)
    want = x.double().numpy() + y_sh + y_w
    assert np.allclose(res["out"], want, rtol=0, atol=1e-12 * np.abs(want).max())
    # the bf16 output is the round-to-nearest-even of the double output
    assert np.array_equal(res["out_bf16"], oracle_lib.round_bf16(res["out"]))
    rb = torch.from_numpy(res["out"]).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(res["out_bf16"], rb)


def test_layer_is_gate_weighted_sum_of_selected_experts(oracle_lib):
    c = TINY
    H, I, Nr, Kr = c["H"], c["I"], c["Nr"], c["Kr"]
    cf = oracle_lib.cfg(H, I, Nr, Kr)
    x = gen_x(16, H, 2)
    Wr = gen_router(Nr, H, 2)
    b = gen_bias(Nr, 2)
    experts = [_quant_expert(oracle_lib, e, H, I, 2) for e in range(Nr + 1)]
    res = oracle_lib.forward(cf, x, Wr, b, experts, tokens=np.array([3, 0, 15, 7]))
    idx, gate, gap, _ = oracle_lib.route(cf, x, Wr, b)
    xq, xs = oracle_lib.quant_1x128(x)
    for r, t in enumerate([3, 0, 15, 7]):
        assert np.array_equal(res["idx"][r], idx[t])
        want = x[t].double().numpy() + oracle_lib.expert_ffn(cf, xq[t:t + 1], xs[t:t + 1], *experts[Nr])[0]
        for k in range(Kr):
            want = want + gate[t, k] * oracle_lib.expert_ffn(cf, xq[t:t + 1], xs[t:t + 1], *experts[idx[t, k]])[0]
        assert np.allclose(res["out"][r], want, rtol=0, atol=1e-12 * np.abs(want).max())


def test_forward_reports_missing_expert(oracle_lib):
    c = TINY
    H, I, Nr, Kr = c["H"], c["I"], c["Nr"], c["Kr"]
    cf = oracle_lib.cfg(H, I, Nr, Kr)
    x = gen_x(4, H, 3)
    ex = _quant_expert(oracle_lib, 0, H, I, 3)
    try:
        oracle_lib.forward(cf, x, gen_router(Nr, H, 3), gen_bias(Nr, 3), [ex] * Nr + [None])
    except ValueError:
        return
    raise AssertionError("missing shared expert was not reported")


def test_bias_update_closed_form(oracle_lib):
    Nr, T, Kr = 8, 10, 4
    total = T * Kr  # mean load = 5
    counts = np.array([5, 6, 4, 0, 10, 5, 5, 5], np.int32)
    assert counts.sum() == total
    b = np.array([0.0, 0.01, -0.01, 0.5, -0.5, 1e-4, 0.001, -0.001], np.float32)
    out = oracle_lib.bias_update(b, counts, Nr, total, 0.001)
    g = np.float32(0.001)
    want = b.copy()
    want[1] = np.float32(b[1] - g)
    want[4] = np.float32(b[4] - g)
    want[2] = np.float32(b[2] + g)
    want[3] = np.float32(b[3] + g)
    assert np.array_equal(out, want)
    # fractional mean: 3 tokens x 1 slot over 2 experts -> 1.5 each
    out2 = oracle_lib.bias_update(np.zeros(2, np.float32), np.array([2, 1], np.int32), 2, 3, 0.001)
    assert out2[0] == -g and out2[1] == g


def test_round_bf16_ties_subnormals_and_signs(oracle_lib):
    """The output rounding (bf16, round to nearest, ties to even) on the cases
    random outputs never reach: exact midpoints between neighbouring bf16
    values, values a hair off them, subnormals, signed zeros."""
    rng = np.random.default_rng(3)
    # random normal bf16 values b and their upper neighbours
    bits = rng.integers(0x0080, 0x7F00, size=4000).astype(np.uint16)  # positive normals
    lo = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    hi = ((bits.astype(np.uint32) + 1) << 16).view(np.float32).astype(np.float64)
    mid = (lo + hi) / 2  # exact in double
    even = np.where(bits % 2 == 0, bits, bits + 1).astype(np.uint16)
    got = oracle_lib.round_bf16(np.concatenate([mid, -mid]))
    assert np.array_equal(got[:4000], even)
    assert np.array_equal(got[4000:], even | np.uint16(0x8000))
    # a hair above / below the midpoint goes to the nearer neighbour
    up = oracle_lib.round_bf16(np.nextafter(mid, np.inf))
    down = oracle_lib.round_bf16(np.nextafter(mid, -np.inf))
    assert np.array_equal(up, (bits + 1).astype(np.uint16)) and np.array_equal(down, bits)
    # subnormals (below 2^-126) and zeros, against the library cast
    sub = np.concatenate([rng.uniform(-2.0 ** -126, 2.0 ** -126, 2000), [0.0, -0.0, 2.0 ** -133, -2.0 ** -134]])
    ref = torch.from_numpy(sub).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle_lib.round_bf16(sub), ref)
