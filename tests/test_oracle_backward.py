"""Pins of the backward oracle of one FP8 expert FFN (``oracle/backward.py``).

The pages fix only "E4M3 for all tensors" ("DeepSeek-V3 Technischer
Bericht", Kernideen, FP8 bullet); the tile orientation of the backward GEMMs
is a reading (1x128 along each GEMM's contraction: rows for dgrad, 128x1
tiles along tokens for wgrad).  What pins it here:
* a dense double-precision gradient of the SwiGLU FFN written in this file,
  itself pinned by central finite differences;
* the FP8 gradients against that dense gradient of the dequantized weights
  (quantization error only: a transposed operand, a swapped W1/W3 or a wrong
  silu' is far outside the bound);
* exact properties: scaling dY by 2^j scales every gradient by exactly 2^j;
  with one token every 128x1 tile holds one value, so the weight gradients
  are outer products to FP32 precision; a ragged token tail equals zero
  padding; the 128x1 tiles run along tokens.
"""
import numpy as np
import pytest
import torch

import moe_synth as S


@pytest.fixture(scope="module")
def bw(oracle_lib):
    import oracle.backward as B
    return B


def dense_backward(x, dy, W1, W3, W2):
    """Analytic gradient of Y = (silu(x W1^T) * (x W3^T)) W2^T, double."""
    G = x @ W1.T
    U = x @ W3.T
    sg = 1.0 / (1.0 + np.exp(-G))
    a = G * sg
    h = a * U
    dh = dy @ W2
    dG = dh * U * sg * (1.0 + G * (1.0 - sg))
    dU = dh * a
    return dict(dx=dG @ W1 + dU @ W3, dW1=dG.T @ x, dW3=dU.T @ x, dW2=dy.T @ h, h=h, G=G, U=U, dh=dh)


def _dense_loss(x, dy, W1, W3, W2):
    G = x @ W1.T
    h = G / (1.0 + np.exp(-G)) * (x @ W3.T)
    return float(np.sum(dy * (h @ W2.T)))


def test_dense_reference_matches_finite_differences():
    rng = np.random.default_rng(0)
    rows, H, I = 5, 7, 6
    x, dy = rng.normal(size=(rows, H)), rng.normal(size=(rows, H))
    W1, W3, W2 = rng.normal(size=(I, H)) * 0.5, rng.normal(size=(I, H)) * 0.5, rng.normal(size=(H, I)) * 0.5
    g = dense_backward(x, dy, W1, W3, W2)
    eps = 1e-6
    for name, arr in (("dx", x), ("dW1", W1), ("dW3", W3), ("dW2", W2)):
        num = np.zeros_like(arr)
        for ij in np.ndindex(arr.shape):
            old = arr[ij]
            arr[ij] = old + eps
            lp = _dense_loss(x, dy, W1, W3, W2)
            arr[ij] = old - eps
            lm = _dense_loss(x, dy, W1, W3, W2)
            arr[ij] = old
            num[ij] = (lp - lm) / (2 * eps)
        np.testing.assert_allclose(g[name], num, rtol=1e-6, atol=1e-7, err_msg=name)


def _skew_blocks(w: torch.Tensor, seed: int) -> torch.Tensor:
    """Each 128x128 block times its own power of two in [1/4, 4] (exact in
    bf16), so that a block scale applied to the wrong block is off by >= 2x."""
    f = 2.0 ** np.random.default_rng(seed).integers(-2, 3, size=(w.shape[0] // 128, w.shape[1] // 128))
    return (w.float() * torch.from_numpy(np.kron(f, np.ones((128, 128)))).float()).to(torch.bfloat16)


def _problem(oracle_lib, rows, H=256, I=256, seed=0, w_std=None):
    x = S.gen_x(rows, H, seed)
    dy = S.normal_bf16((rows, H), 1.0, seed + 1000)
    if w_std is None:
        w13, w2 = S.gen_expert(seed % 7, H, I, seed)
    else:  # larger, block-skewed weights: G spreads over the nonlinear part of silu
        w13 = _skew_blocks(S.normal_bf16((2 * I, H), w_std, seed + 2000), seed + 4000)
        w2 = _skew_blocks(S.normal_bf16((H, I), w_std, seed + 3000), seed + 5000)
    W13q, s13 = oracle_lib.quant_128x128(w13)
    W2q, s2 = oracle_lib.quant_128x128(w2)
    return x, dy, W13q, s13, W2q, s2


def _rel(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


@pytest.mark.parametrize("w_std,I", [(None, 256), (0.1, 384)])
def test_fp8_backward_tracks_the_dense_gradient(oracle_lib, bw, w_std, I):
    x, dy, W13q, s13, W2q, s2 = _problem(oracle_lib, 256, I=I, w_std=w_std)
    I = W13q.shape[0] // 2
    W13 = oracle_lib.dequant(W13q, s13, 128)
    W2 = oracle_lib.dequant(W2q, s2, 128)
    xd, dyd = x.double().numpy(), dy.double().numpy()
    ref = dense_backward(xd, dyd, W13[:I], W13[I:], W2)
    got = bw.expert_backward(x, dy, W13q, s13, W2q, s2)
    dW13_ref = np.concatenate([ref["dW1"], ref["dW3"]])
    # E4M3 keeps 3 mantissa bits (relative step up to 2^-4 per element); a
    # GEMM of two quantized operands lands at a few % rel-Frobenius, and the
    # chain dY -> dh -> dG, dU -> dx quantizes twice
    errs = dict(G=_rel(got["G"], ref["G"]), h=_rel(got["h"], ref["h"]), dh=_rel(got["dh"], ref["dh"]),
                dx=_rel(got["dx"], ref["dx"]), dW13=_rel(got["dW13"], dW13_ref), dW2=_rel(got["dW2"], ref["dW2"]))
    print("rel-Frobenius vs dense:", {k: f"{v:.3f}" for k, v in errs.items()})
    assert max(errs.values()) < 0.12, errs
    if w_std is None:
        return
    # with G spread over silu's nonlinear part the bound separates plausible
    # mistakes: W1/W3 swapped, a transposed weight gradient, or silu'
    # replaced by sigma
    bad = dense_backward(xd, dyd, W13[I:], W13[:I], W2)
    assert _rel(got["dx"], bad["dx"]) > 0.5
    assert _rel(got["dW2"], (dyd.T @ ref["h"][:, ::-1])) > 0.5
    sg = 1.0 / (1.0 + np.exp(-ref["G"]))
    dG_wrong = ref["dh"] * ref["U"] * sg
    assert _rel(got["dG"], dG_wrong) > 0.12


def test_power_of_two_scaling_of_dy_scales_every_gradient_exactly(oracle_lib, bw):
    x, dy, W13q, s13, W2q, s2 = _problem(oracle_lib, 200, seed=3)
    a = bw.expert_backward(x, dy, W13q, s13, W2q, s2)
    b = bw.expert_backward(x, (dy.float() * 8.0).to(torch.bfloat16), W13q, s13, W2q, s2)
    for k in ("dx", "dW13", "dW2", "dh", "dG", "dU"):
        assert np.array_equal(b[k], 8.0 * a[k]), k
    for k in ("G", "U", "h"):
        assert np.array_equal(b[k], a[k]), k


def test_single_token_weight_gradients_are_outer_products(oracle_lib, bw):
    # one token: each 128x1 tile holds one value, which quantizes to +-448
    # times its scale, i.e. back to itself up to FP32 rounding of the scale
    x, dy, W13q, s13, W2q, s2 = _problem(oracle_lib, 1, seed=4)
    r = bw.expert_backward(x, dy, W13q, s13, W2q, s2)
    xd, dyd = x.double().numpy(), dy.double().numpy()
    np.testing.assert_allclose(r["dW2"], dyd.T @ r["h"], rtol=1e-6, atol=0)
    np.testing.assert_allclose(r["dW13"], np.concatenate([r["dG"].T @ xd, r["dU"].T @ xd]), rtol=1e-6, atol=0)


def test_ragged_token_tail_equals_zero_padding(oracle_lib, bw):
    x, dy, W13q, s13, W2q, s2 = _problem(oracle_lib, 200, seed=5)
    pad = lambda t: torch.cat([t, torch.zeros((56, t.shape[1]), dtype=t.dtype)])  # noqa: E731
    a = bw.expert_backward(x, dy, W13q, s13, W2q, s2)
    b = bw.expert_backward(pad(x), pad(dy), W13q, s13, W2q, s2)
    assert np.array_equal(a["dW13"], b["dW13"]) and np.array_equal(a["dW2"], b["dW2"])
    assert np.array_equal(a["dx"], b["dx"][:200])


def test_wgrad_tiles_run_along_tokens(oracle_lib, bw):
    rows, cols = 300, 256
    x = S.normal_bf16((rows, cols), 1.0, 6)
    q0, s0 = bw.quant_128x1_bf16(x)
    assert s0.shape == (3, cols)
    # the scale of a tile is the amax of its (up to) 128 tokens over 448
    xf = np.abs(x.float().numpy())
    for tb in range(3):
        amax = xf[tb * 128:(tb + 1) * 128].max(axis=0).astype(np.float32)
        assert np.array_equal(s0[tb], amax / np.float32(448.0))
    y = x.clone()
    y[260, 17] = 50.0  # a new amax in tile (tokens 256..299, column 17)
    q1, s1 = bw.quant_128x1_bf16(y)
    changed = np.argwhere(s1 != s0)
    assert changed.tolist() == [[2, 17]]
    diff = np.argwhere(q1 != q0)
    assert (diff[:, 1] == 17).all() and (diff[:, 0] >= 256).all()


def test_rows_scaled_gemm_matches_dense_dequantized(oracle_lib, bw):
    rng = np.random.default_rng(7)
    M, N, K = 24, 16, 300
    qa = rng.integers(0, 256, size=(M, K)).astype(np.uint8)
    qb = rng.integers(0, 256, size=(N, K)).astype(np.uint8)
    qa[(qa & 0x7F) == 0x7F] = 0  # no NaN codes
    qb[(qb & 0x7F) == 0x7F] = 0
    sa = rng.uniform(0.5, 2.0, size=(M, 3)).astype(np.float32)
    sb = rng.uniform(0.5, 2.0, size=(N, 3)).astype(np.float32)
    got = bw.rows_scaled_gemm(qa, sa, qb, sb)
    dec = oracle_lib.e4m3_decode_table()
    A = dec[qa] * np.repeat(sa.astype(np.float64), 128, axis=1)[:, :K]
    B = dec[qb] * np.repeat(sb.astype(np.float64), 128, axis=1)[:, :K]
    np.testing.assert_allclose(got, A @ B.T, rtol=1e-12, atol=1e-9)


# ------------------------------------------------------------ layer level
def _layer_problem(oracle_lib, T=96, seed=0, zero_weights=False):
    cfg = dict(S.TINY)
    H, I, Nr, Kr = cfg["H"], cfg["I"], cfg["Nr"], cfg["Kr"]
    x = S.gen_x(T, H, seed)
    wr = S.gen_router(Nr, H, seed)
    bias = S.gen_bias(Nr, seed)
    dout = S.normal_bf16((T, H), 1.0, seed + 77)
    experts = []
    for e in range(Nr + 1):
        w13, w2 = S.gen_expert(e, H, I, seed)
        if zero_weights:
            w13, w2 = torch.zeros_like(w13), torch.zeros_like(w2)
        a, sa = oracle_lib.quant_128x128(w13)
        b, sb = oracle_lib.quant_128x128(w2)
        experts.append((a, sa, b, sb))
    cf = oracle_lib.cfg(H, I, Nr, Kr)
    return cf, x, wr, bias, dout, experts


def test_layer_backward_residual_path_is_exact(oracle_lib, bw):
    cf, x, wr, bias, dout, experts = _layer_problem(oracle_lib, zero_weights=True)
    r = bw.layer_backward(cf, x, wr, bias, experts, dout)
    assert np.array_equal(r["dx"], dout.double().numpy())
    assert all(not w.any() for w in list(r["dW13"].values()) + list(r["dW2"].values()))


def test_layer_backward_scales_exactly_with_dout(oracle_lib, bw):
    cf, x, wr, bias, dout, experts = _layer_problem(oracle_lib, seed=1)
    a = bw.layer_backward(cf, x, wr, bias, experts, dout)
    b = bw.layer_backward(cf, x, wr, bias, experts, (dout.float() * 0.25).to(torch.bfloat16))
    # every term (residual, each expert's dx) and the FP32 rounding of their
    # sum scale exactly by a power of two
    assert np.array_equal(b["dx"], 0.25 * a["dx"])
    for e in a["dW13"]:
        assert np.array_equal(b["dW13"][e], 0.25 * a["dW13"][e]) and np.array_equal(b["dW2"][e], 0.25 * a["dW2"][e])


def test_layer_backward_tracks_the_dense_layer_gradient(oracle_lib, bw):
    cf, x, wr, bias, dout, experts = _layer_problem(oracle_lib, T=128, seed=2)
    r = bw.layer_backward(cf, x, wr, bias, experts, dout)
    I, Nr = S.TINY["I"], S.TINY["Nr"]
    xd, dd = x.double().numpy(), dout.double().numpy()

    def dense(e):
        W13 = oracle_lib.dequant(experts[e][0], experts[e][1], 128)
        return W13[:I], W13[I:], oracle_lib.dequant(experts[e][2], experts[e][3], 128)

    dx = dd + dense_backward(xd, dd, *dense(Nr))["dx"]
    used = sorted(set(r["idx"].reshape(-1).tolist()))
    assert sorted(k for k in r["dW13"] if k < Nr) == used and Nr in r["dW13"]
    rel_w = []
    for e in used:
        toks, slots = np.nonzero(r["idx"] == e)
        g = r["gate"][toks, slots][:, None]
        ref = dense_backward(xd[toks], g * dd[toks], *dense(e))
        dx[toks] += ref["dx"]
        rel_w.append(_rel(r["dW2"][e], ref["dW2"]))
        rel_w.append(_rel(r["dW13"][e], np.concatenate([ref["dW1"], ref["dW3"]])))
    # residual excluded from the comparison so it does not mask the experts' part
    rel = _rel(r["dx"] - dd, dx - dd)
    print(f"layer dx rel-Frobenius {rel:.3f}; weight gradients max {max(rel_w):.3f}")
    assert rel < 0.12 and max(rel_w) < 0.15


def test_gate_placement(oracle_lib, bw):
    # dY = g D.  A power-of-two gate is exact in every step, so handing the
    # gate to expert_backward must give bitwise the gradients of the scaled
    # D (a dropped gate, or one applied twice, differs by 2x).  A general
    # gate moves only the rounding of g D out of the dgrad's codes.
    x, dy, W13q, s13, W2q, s2 = _problem(oracle_lib, 200, seed=8)
    rows = dy.shape[0]
    g = 2.0 ** np.random.default_rng(8).integers(-3, 1, size=rows)
    a = bw.expert_backward(x, dy, W13q, s13, W2q, s2, gate=g)
    b = bw.expert_backward(x, (dy.float() * torch.from_numpy(g).float()[:, None]).numpy(), W13q, s13, W2q, s2)
    for k in ("dx", "dW13", "dh", "dG", "dU"):
        assert np.array_equal(a[k], b[k]), k
    assert np.array_equal(a["gh"], g[:, None] * a["h"])
    # in dW2 the gate moves between the operands of 128x1 tiles with mixed
    # gates, which changes their codes; with one gate for every row it does not
    assert _rel(a["dW2"], b["dW2"]) < 0.1
    a = bw.expert_backward(x, dy, W13q, s13, W2q, s2, gate=np.full(rows, 0.25))
    b = bw.expert_backward(x, (dy.float() * 0.25).numpy(), W13q, s13, W2q, s2)
    assert np.array_equal(a["dW2"], b["dW2"])
    g = np.random.default_rng(9).uniform(0.05, 0.6, size=rows)
    a = bw.expert_backward(x, dy, W13q, s13, W2q, s2, gate=g)
    b = bw.expert_backward(x, (dy.float() * torch.from_numpy(g).float()[:, None]).numpy(), W13q, s13, W2q, s2)
    for k in ("dx", "dW13", "dh"):
        assert _rel(a[k], b[k]) < 2e-2, k
    assert _rel(a["dW2"], b["dW2"]) < 0.1
    assert np.array_equal(a["G"], b["G"])
