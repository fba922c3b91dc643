"""Full-size parity: the DeepSeek-V3-shaped layer (hidden 7168, intermediate
2048, 256 routed + 1 shared experts, top-8) in the launch configuration the
benchmark times.  Quantization, routing, counts, grouping and weights are
checked over the whole batch; the expert FFNs and the layer output on tokens
the double-precision oracle computes one by one: all 64 decode tokens, and at
prefill and skewed sizes at least 64 tokens chosen so that their rows reach
all four TMEM lane quarters (of both CTAs where tiles run on CTA pairs) and
the most loaded expert (pick_tokens)."""
import numpy as np
import pytest
import torch

import moe_synth as S
from _moe_util import Problem
from test_gpu_layer import check_balance_loss, check_layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def m():
    import sparse_moe_layer_expert_b200 as pkg
    return pkg


@pytest.fixture(scope="module")
def v3_layer(m):
    """One GPU-resident V3 layer (weights generated on the GPU per expert,
    quantized by the library), shared by the full-size tests."""
    cfg = dict(S.PREFILL)
    shape = {k: cfg[k] for k in ("H", "I", "Nr", "Kr", "Ns")}
    seed = 0

    def gen(e):
        return S.gen_expert(e, cfg["H"], cfg["I"], seed, device="cuda")

    wr = S.gen_router(cfg["Nr"], cfg["H"], seed, device="cuda")
    bias = S.gen_bias(cfg["Nr"], seed, "uniform", device="cuda")
    layer = m.MoeLayer.from_generator(shape, gen, wr, bias)
    torch.cuda.synchronize()
    return layer, seed


def pick_tokens(m, layer, prob, n: int, seed: int) -> np.ndarray:
    """Tokens for the per-token FFN comparison, chosen so that their rows
    reach every part of the grouped GEMMs' tiles.  From the chunk table the
    forward leaves in its workspace (each chunk: one expert's rows, up to 128
    per CTA; on CTA pairs up to 256, rows 128.. on the odd CTA): rows in each
    of the four 32-row TMEM lane quarters of each CTA position, routed and
    shared; rows of the most loaded expert; the first and the last token;
    then seeded random tokens up to n."""
    T, Kr, Nr = prob.T, prob.cfg["Kr"], prob.cfg["Nr"]
    layer.forward(prob.x)
    layer.check()
    ws, L = layer.workspace(T), layer.layout(T)
    idx = m.ws_view(ws, L, "idx", torch.int32, (T, Kr)).cpu().numpy()
    pos = m.ws_view(ws, L, "pos", torch.int32, (T, Kr)).cpu().numpy()
    off = m.ws_view(ws, L, "offsets", torch.int32, (Nr + 1,)).cpu().numpy()
    nch = int(m.ws_view(ws, L, "meta", torch.int32, (4,)).cpu().numpy()[0])
    chunks = m.ws_view(ws, L, "chunks", torch.int32, (nch, 4)).cpu().numpy()
    R = T * Kr
    token_of_row = np.empty(R + T, np.int64)
    token_of_row[pos.reshape(-1)] = np.repeat(np.arange(T), Kr)
    token_of_row[R:] = np.arange(T)
    want = {}
    for _, _, out_row, rows in chunks:
        rows &= 0xFFFF  # the expert's chunk count sits in the high bits
        for r in range(rows):
            row = out_row + r
            key = ("shared" if row >= R else "routed", r >= 128, (r % 128) // 32)
            want.setdefault(key, []).append(int(token_of_row[row]))
    rng = np.random.default_rng(seed)
    chosen = {0, T - 1}
    for key in sorted(want):
        cand = want[key]
        chosen.update(int(c) for c in rng.choice(cand, min(2, len(cand)), replace=False))
    hot = int(np.argmax(np.diff(off)))
    hot_tokens = np.nonzero((idx == hot).any(axis=1))[0]
    chosen.update(int(c) for c in rng.choice(hot_tokens, min(4, len(hot_tokens)), replace=False))
    rest = np.setdiff1d(np.arange(T), np.array(sorted(chosen)))
    extra = max(0, n - len(chosen))
    chosen.update(int(c) for c in rng.choice(rest, min(extra, len(rest)), replace=False))
    return np.array(sorted(chosen))


def _problem(cfg, T, seed, layer, bias_kind):
    prob = Problem(cfg, T, seed=seed, device="cuda")
    # the layer's weights and router come from seed 0; only x differs per test
    prob.seed = 0
    prob.wr = layer.wr
    prob.bias = layer.bias.clone()
    if bias_kind == "zero":
        prob.bias.zero_()
    layer.bias.copy_(prob.bias)
    prob.x = S.gen_x(T, cfg["H"], seed, device="cuda")
    return prob


def test_v3_decode_layer(m, oracle_lib, v3_layer):
    layer, _ = v3_layer
    prob = _problem(dict(S.DECODE), 64, 11, layer, "zero")
    # every token of the batch
    r = check_layer(m, oracle_lib, prob, layer, tokens=np.arange(64), check_weights=True)
    assert r["counts"].sum() == 64 * 8


def test_v3_prefill_layer(m, oracle_lib, v3_layer):
    layer, _ = v3_layer
    prob = _problem(dict(S.PREFILL), 4096, 12, layer, "uniform")
    toks = pick_tokens(m, layer, prob, 64, 12)
    assert len(toks) >= 64
    r = check_layer(m, oracle_lib, prob, layer, tokens=toks, check_weights=False)
    c = r["counts"]
    print(f"prefill load: max {c.max()} mean {c.mean():.1f} min {c.min()} empty {(c == 0).sum()}")
    # the sequence-wise balance loss: one 4096-token sequence, and four of 1024
    loss = check_balance_loss(oracle_lib, prob, layer, r, 4096)
    check_balance_loss(oracle_lib, prob, layer, r, 1024)
    print(f"prefill sequence-wise balance loss (alpha 1e-4): {loss[0]:.6e}")


def test_v3_skewed_layer(m, oracle_lib, v3_layer):
    """The skewed configuration at full size: 16384 tokens of the centroid-
    mixture input, group-limited routing (8 groups of 32 experts, top-4
    groups), zero bias; the V3 weights of the shared fixture, routed through a
    layer object configured for group-limited routing."""
    base, _ = v3_layer
    cfg = dict(S.SKEWED)
    shape = {k: cfg[k] for k in ("H", "I", "Nr", "Kr", "Ns", "n_groups", "topk_groups")}
    layer = m.MoeLayer(shape)
    layer.w13, layer.s13, layer.w2, layer.s2 = base.w13, base.s13, base.w2, base.s2  # same weights, no copy
    T = cfg["T"]
    prob = Problem(cfg, T, seed=13, device="cuda")  # mixture input (the configuration's x)
    prob.seed = 0                                    # weights and router of the fixture (seed 0)
    prob.wr = base.wr
    prob.bias = torch.zeros(cfg["Nr"], dtype=torch.float32, device="cuda")
    layer.set_router(prob.wr, prob.bias)
    toks = pick_tokens(m, layer, prob, 64, 13)
    assert len(toks) >= 64
    r = check_layer(m, oracle_lib, prob, layer, tokens=toks, check_weights=False)
    c = r["counts"]
    print(f"skewed load: max {c.max()} mean {c.mean():.1f} max/mean {c.max() / c.mean():.2f}")
    assert c.max() >= 4 * c.mean()  # the configuration's imbalance (max/mean load >= 4)
    loss = check_balance_loss(oracle_lib, prob, layer, r, 4096)
    print(f"skewed sequence-wise balance loss (alpha 1e-4), four 4096-token sequences: {loss}")


@pytest.fixture(scope="module")
def v3_layer_pow2(m):
    """The same V3 layer with power-of-two scales (block-scaled GEMM path)."""
    cfg = dict(S.PREFILL)
    shape = {k: cfg[k] for k in ("H", "I", "Nr", "Kr", "Ns")}
    shape["scale_mode"] = m.MOE_SCALE_POW2
    seed = 0

    def gen(e):
        return S.gen_expert(e, cfg["H"], cfg["I"], seed, device="cuda")

    wr = S.gen_router(cfg["Nr"], cfg["H"], seed, device="cuda")
    bias = S.gen_bias(cfg["Nr"], seed, "uniform", device="cuda")
    layer = m.MoeLayer.from_generator(shape, gen, wr, bias)
    torch.cuda.synchronize()
    return layer, seed


def test_v3_prefill_layer_pow2(m, oracle_lib, v3_layer_pow2):
    layer, _ = v3_layer_pow2
    prob = _problem(dict(S.PREFILL, scale_mode=1), 4096, 12, layer, "uniform")
    rng = np.random.default_rng(14)
    toks = np.sort(rng.choice(4096, 16, replace=False))
    check_layer(m, oracle_lib, prob, layer, tokens=toks, check_weights=True)


def test_v3_decode_layer_pow2(m, oracle_lib, v3_layer_pow2):
    layer, _ = v3_layer_pow2
    prob = _problem(dict(S.DECODE, scale_mode=1), 64, 11, layer, "zero")
    r = check_layer(m, oracle_lib, prob, layer, tokens=np.array([0, 9, 31, 63]), check_weights=False)
    assert r["counts"].sum() == 64 * 8


def test_v3_skewed_layer_pow2(m, oracle_lib, v3_layer_pow2):
    """The skewed configuration at full size in the power-of-two scale mode
    (the block-scaled GEMMs on hot experts with thousands of rows)."""
    base, _ = v3_layer_pow2
    cfg = dict(S.SKEWED, scale_mode=1)
    shape = {k: cfg[k] for k in ("H", "I", "Nr", "Kr", "Ns", "n_groups", "topk_groups", "scale_mode")}
    layer = m.MoeLayer(shape)
    layer.w13, layer.s13, layer.w2, layer.s2 = base.w13, base.s13, base.w2, base.s2  # same weights, no copy
    T = cfg["T"]
    prob = Problem(cfg, T, seed=15, device="cuda")
    prob.seed = 0
    prob.wr = base.wr
    prob.bias = torch.zeros(cfg["Nr"], dtype=torch.float32, device="cuda")
    layer.set_router(prob.wr, prob.bias)
    rng = np.random.default_rng(15)
    toks = np.sort(rng.choice(T, 16, replace=False))
    r = check_layer(m, oracle_lib, prob, layer, tokens=toks, check_weights=False)
    c = r["counts"]
    assert c.max() >= 4 * c.mean()


@pytest.fixture
def tall(m):
    m.moe_set_gemm_variant(m.MOE_GEMM_TALL)
    yield m
    m.moe_set_gemm_variant(m.MOE_GEMM_AUTO)


def test_v3_prefill_layer_tall(tall, oracle_lib, v3_layer):
    # tall tiles (up to 256 rows per weight pass): rows 128.. land in the
    # second promotion warpgroup; pick_tokens covers every lane quarter of both
    m = tall
    layer, _ = v3_layer
    prob = _problem(dict(S.PREFILL), 4096, 14, layer, "uniform")
    assert m.moe_gemm_kernel_for(layer.cfg, 4096) == m.MOE_GEMM_TALL
    toks = pick_tokens(m, layer, prob, 64, 14)
    assert len(toks) >= 64
    check_layer(m, oracle_lib, prob, layer, tokens=toks, check_weights=False)


def test_v3_decode_layer_tall(tall, oracle_lib, v3_layer):
    m = tall
    layer, _ = v3_layer
    prob = _problem(dict(S.DECODE), 64, 15, layer, "zero")
    check_layer(m, oracle_lib, prob, layer, tokens=np.arange(64), check_weights=False)


def test_v3_expert_parallel_emulated(m, oracle_lib, v3_layer):
    """The expert-parallel forward of 8 ranks x 256 tokens on the V3 layer, all
    ranks' kernels on this GPU (exchanges as device copies), against the
    oracle's single-device layer on 8 sampled tokens per rank (off near-ties).
    The reading (R-EP) returns each destination rank's partial sum and the
    shared expert's output as bf16, so the max bound of an element also takes
    half a bf16 ulp of each such term, from the oracle's own per-expert
    outputs; the relative Frobenius bound is the stated one."""
    from sparse_moe_layer_expert_b200.ep import LibraryOps, forward_local
    from _moe_util import half_ulp_bf16, assert_close, oracle_cfg, NEAR_TIE
    from test_gpu_layer import h_tie_allowance
    dec = oracle_lib.e4m3_decode_table()
    layer, _ = v3_layer
    W, T = 8, 256
    cfg = dict(S.PREFILL)
    prob = _problem(cfg, T, 21, layer, "uniform")
    layer.bias.copy_(prob.bias)
    ops = [LibraryOps(layer, W, r) for r in range(W)]
    xs = [S.gen_x(T, cfg["H"], 300 + r, device="cuda") for r in range(W)]
    outs = forward_local(ops, xs, m.MOE_DTYPE_F32)
    layer.check()
    ocf = oracle_cfg(oracle_lib, cfg)
    Nr, per = cfg["Nr"], cfg["Nr"] // W
    experts = {}
    rng = np.random.default_rng(21)
    for r in range(W):
        x = xs[r].cpu()
        oi, og, gap, _ = oracle_lib.route(ocf, x, prob.wr, prob.bias)
        toks = np.sort(rng.choice(np.nonzero(gap >= NEAR_TIE)[0], 8, replace=False))
        for e in set(oi[toks].reshape(-1).tolist()) | {Nr}:
            if e not in experts:
                experts[e] = prob.oracle_expert(oracle_lib, e)
        res = oracle_lib.forward(ocf, x, prob.wr, prob.bias, [experts.get(e) for e in range(Nr + 1)], tokens=toks)
        assert np.array_equal(res["idx"], oi[toks])
        xq, xsc = oracle_lib.quant_1x128(x[torch.as_tensor(toks)])
        allow = np.zeros((len(toks), cfg["H"]))
        for i, t in enumerate(toks):
            # (and, as in every layer test, what codes of h at a rounding
            # near-tie can move each expert's output by)
            ysh, hsh, _, hssh = oracle_lib.expert_ffn(ocf, xq[i:i + 1], xsc[i:i + 1], *experts[Nr], want_h=True)
            allow[i] += half_ulp_bf16(ysh[0]) + h_tie_allowance(dec, hsh[0], hssh[0], experts[Nr][2], experts[Nr][3])
            part = {}
            for k in range(cfg["Kr"]):
                e = int(oi[t, k])
                y, h, _, hs = oracle_lib.expert_ffn(ocf, xq[i:i + 1], xsc[i:i + 1], *experts[e], want_h=True)
                part[e // per] = part.get(e // per, 0.0) + og[t, k] * y[0]
                allow[i] += og[t, k] * h_tie_allowance(dec, h[0], hs[0], experts[e][2], experts[e][3])
            for d in part:
                allow[i] += half_ulp_bf16(part[d])
        got = outs[r].cpu().numpy().astype(np.float64)[toks]
        assert_close(got, res["out"], what=f"expert-parallel V3 output, rank {r} of {W}", tie_allow=allow)
