"""GPU parity of the FP8 backward of the expert FFNs (moe_backward, routing
held fixed) against the oracle's layer backward (oracle/backward.py): the
input gradient dx and every expert's weight gradients dW13, dW2, on the small
configuration (all tokens; experts with several 128-token tiles and ragged
tails) and on one expert at full DeepSeek-V3 size ("DeepSeek-V3 Technischer
Bericht", Kernideen, FP8 bullet: E4M3 for all tensors; the backward tile
orientation is the reading the oracle documents).  Tolerance: the layer's
stated bound (relative Frobenius error 2e-3, max |diff| 1e-2 rms) on every
FP32 output, the max bound widened by what codes of the FP32 intermediates
dG, dU and g*h at a rounding near-tie can change (either code is a correct
result there; near_tie_steps); the intermediates themselves agree to FP32
rounding."""
import numpy as np
import pytest
import torch

import moe_synth as S
from _moe_util import NEAR_TIE, Problem, assert_close, near_tie_steps, oracle_cfg, tiles_128x1, tiles_1x128
from test_gpu_layer import build_gpu_layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def m():
    import sparse_moe_layer_expert_b200 as pkg
    return pkg


def expert_tie_allowance(oracle_lib, OB, dec, r, x_rows, d_rows, W13q, s13):
    """What codes at a rounding near-tie of the FP32 intermediates dG, dU
    (1x128 along I for dx, 128x1 along tokens for dW13) and g*h (128x1 for
    dW2) can change: per dx row [rows, H], dW13 [2I, H] and dW2 [H, I]
    (near_tie_steps).  The other operand of each GEMM is the oracle's:
    the dequantized weights, the 128x1-quantized x and dout rows."""
    I = r["dG"].shape[1]
    rows = r["dG"].shape[0]
    H = W13q.shape[1]
    W = np.asarray(W13q)
    s13 = np.asarray(s13, np.float64)
    dx_a = np.zeros((rows, H))
    for half, name in ((0, "dG"), (1, "dU")):
        v = r[name].astype(np.float32)
        _, s1 = oracle_lib.quant_1x128_f32(v)
        st = near_tie_steps(v, tiles_1x128(s1), dec)
        for p, i in zip(*np.nonzero(st)):
            row = half * I + i
            dx_a[p] += st[p, i] * np.abs(dec[W[row]] * np.repeat(s13[row // 128], 128))
    xq, xs = OB.quant_128x1_bf16(x_rows)
    xd = np.abs(dec[xq] * tiles_128x1(xs, rows))
    dW13_a = np.zeros((2 * I, H))
    for half, name in ((0, "dG"), (1, "dU")):
        v = r[name].astype(np.float32)
        _, sc = OB.quant_128x1_f32(v)
        st = near_tie_steps(v, tiles_128x1(sc, rows), dec)
        for t, i in zip(*np.nonzero(st)):
            dW13_a[half * I + i] += st[t, i] * xd[t]
    dq, ds = OB.quant_128x1_f32(np.ascontiguousarray(d_rows, np.float32))
    dd = np.abs(dec[dq] * tiles_128x1(ds, rows))
    v = r["gh"].astype(np.float32)
    _, sc = OB.quant_128x1_f32(v)
    st = near_tie_steps(v, tiles_128x1(sc, rows), dec)
    dW2_a = np.zeros((H, I))
    for t, i in zip(*np.nonzero(st)):
        dW2_a[:, i] += st[t, i] * dd[t]
    return dx_a, dW13_a, dW2_a


def run_backward_case(m, oracle_lib, cfg, T, seed, bias_shift=None, zero_dout=0):
    import oracle.backward as OB
    prob = Problem(cfg, T, seed=seed)
    if bias_shift is not None:
        prob.bias = prob.bias.clone()
        prob.bias[:bias_shift] += 1.0
    layer = build_gpu_layer(m, prob)
    x = prob.x.cuda()
    idx_out = torch.empty((T, cfg["Kr"]), dtype=torch.int32, device="cuda")
    layer.forward(x, idx_out=idx_out)
    dout = S.gen_x(T, cfg["H"], seed + 1000)
    if zero_dout:
        dout[:zero_dout] = 0
    dx, dW13, dW2 = layer.backward(x, dout.cuda())
    layer.check()
    experts = [prob.oracle_expert(oracle_lib, e) for e in range(prob.E)]
    ocf = oracle_cfg(oracle_lib, cfg)
    ref = OB.layer_backward(ocf, prob.x, prob.wr, prob.bias, experts, dout, details=True)
    # the same routing on both sides (the configurations are chosen without near-ties)
    assert (ref["gap"] >= NEAR_TIE).all()
    got_idx = idx_out.cpu().numpy()
    for t in range(T):
        assert set(got_idx[t].tolist()) == set(ref["idx"][t].tolist()), t
    H, I, Kr, Ns = cfg["H"], cfg["I"], cfg["Kr"], cfg.get("Ns", 1)
    R, E = T * Kr, prob.E
    RS = R + T * Ns
    # the backward's own intermediates, step by step against the oracle's
    bws, BL = layer.backward_workspace(T), m.moe_backward_workspace_layout(layer.cfg, T)

    def view(name, shape):
        off, nb = BL[name]
        n = int(np.prod(shape))
        assert n * 4 <= nb
        return bws[off:off + 4 * n].view(torch.float32).view(shape).cpu().numpy().astype(np.float64)

    GU, dh, gh, dGU = view("gu", (RS, 2 * I)), view("dh", (RS, I)), view("gh", (RS, I)), view("dgu", (RS, 2 * I))
    ws, L = layer.workspace(T), layer.layout(T)
    offsets = m.ws_view(ws, L, "offsets", torch.int32, (cfg["Nr"] + 1,)).cpu().numpy()
    d32 = dout.float().numpy()
    dec = oracle_lib.e4m3_decode_table()
    dx_allow = np.zeros((T, H))
    w_allow = {}
    msgs, fails = [], []
    for e in sorted(ref["per_expert"].keys()):
        toks, r = ref["per_expert"][e]
        rows = np.arange(offsets[e], offsets[e + 1]) if e < cfg["Nr"] else R + toks
        assert rows.size == toks.size
        # G, U from the same x codes; dh from the same dout codes (the gate on
        # the FP32 result); the rest FP32 elementwise: rounding apart only
        for nm, got, want in (("G", GU[rows, :I], r["G"]), ("U", GU[rows, I:], r["U"]), ("dh", dh[rows], r["dh"]),
                              ("g*h", gh[rows], r["gh"]), ("dG", dGU[rows, :I], r["dG"]),
                              ("dU", dGU[rows, I:], r["dU"])):
            rel = np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30)
            msgs.append(f"expert {e} {nm}: rel-Frobenius {rel:.2e}")
            if not rel < 1e-5:
                fails.append(msgs[-1])
        dxa, w13a, w2a = expert_tie_allowance(oracle_lib, OB, dec, r, prob.x[torch.as_tensor(toks)], d32[toks],
                                              experts[e][0], experts[e][1])
        dx_allow[toks] += dxa
        w_allow[e] = (w13a, w2a)
    print("\n".join(msgs[:60]))
    assert not fails, fails[:10]
    assert_close(dx.cpu().numpy().astype(np.float64), ref["dx"], what="dx", tie_allow=dx_allow)
    dW13_h, dW2_h = dW13.cpu().numpy(), dW2.cpu().numpy()
    used = set(ref["dW13"].keys())
    for e in range(E):
        if e in used:
            assert_close(dW13_h[e].astype(np.float64), ref["dW13"][e], what=f"dW13 of expert {e}",
                         tie_allow=w_allow[e][0])
            assert_close(dW2_h[e].astype(np.float64), ref["dW2"][e], what=f"dW2 of expert {e}",
                         tie_allow=w_allow[e][1])
        else:
            assert not dW13_h[e].any() and not dW2_h[e].any(), f"expert {e} has no token but a gradient"
    if zero_dout:
        assert not dx.cpu()[:zero_dout].any(), "a token with zero dout has a nonzero dx"
    return ref


def test_backward_tiny(m, oracle_lib):
    run_backward_case(m, oracle_lib, dict(S.TINY), 256, 0)


def test_backward_tiny_multi_tile_experts(m, oracle_lib):
    # every token picks experts 0..K_r-1: each holds T = 300 rows, three
    # 128-token tiles of the weight gradients (the last one 44 rows)
    ref = run_backward_case(m, oracle_lib, dict(S.TINY), 300, 3, bias_shift=S.TINY["Kr"])
    assert set(ref["dW13"].keys()) == set(range(S.TINY["Kr"])) | {S.TINY["Nr"]}


def test_backward_zero_dout_tokens(m, oracle_lib):
    # every token picks experts 0..K_r-1 and the first 128 tokens carry a zero
    # dout: their dh, dG, dU and dx are exactly zero, and the first 128-token
    # tile of each expert's dG|dU operand is all zero (the 128x1 quantizer's
    # zero-scale path)
    run_backward_case(m, oracle_lib, dict(S.TINY), 300, 5, bias_shift=S.TINY["Kr"], zero_dout=128)


def test_backward_tiny_ragged_no_shared(m, oracle_lib):
    run_backward_case(m, oracle_lib, dict(S.TINY, Ns=0), 77, 4)


def test_backward_full_size_expert(m, oracle_lib):
    # one V3-sized expert (H = 7168, I = 2048) on 300 tokens: a layer with a
    # single routed expert selected by every token (gate 1) and no shared one
    cfg = dict(H=7168, I=2048, Nr=1, Kr=1, Ns=0, n_groups=0, topk_groups=0, bias="uniform", x="normal")
    run_backward_case(m, oracle_lib, cfg, 300, 5)


def test_backward_rejects_pow2_and_small_workspace(m):
    prob = Problem(dict(S.TINY, scale_mode=1), 8, seed=6)
    layer = build_gpu_layer(m, prob)
    x = prob.x.cuda()
    layer.forward(x)
    with pytest.raises(m.MoeError) as e:
        layer.backward(x, x)
    assert e.value.status == m.MOE_ERR_NOT_IMPLEMENTED
    prob = Problem(S.TINY, 8, seed=6)
    layer = build_gpu_layer(m, prob)
    layer.forward(x)
    wt = m.moe_transpose_weights(layer.cfg, layer.weights())
    with pytest.raises(m.MoeError) as e:
        m.moe_backward(layer.cfg, layer.weights(), wt, x, x, layer.workspace(8),
                       ws=torch.empty(1024, dtype=torch.uint8, device="cuda"), err=layer.err)
    assert e.value.status == m.MOE_ERR_WORKSPACE_TOO_SMALL


def test_backward_profile_events(m):
    """With 7 + 9 event handles the backward marks its stages on the stream:
    every stage time is non-negative and they add up to the whole call."""
    prob = Problem(S.TINY, 300, seed=9)
    layer = build_gpu_layer(m, prob)
    x = prob.x.cuda()
    layer.forward(x)
    dout = S.gen_x(300, S.TINY["H"], 1009).cuda()
    layer.backward(x, dout)  # set-up (transposed weights) outside the measured call
    nf, nb = m.MOE_PROFILE_EVENTS, m.MOE_PROFILE_BWD_EVENTS
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(nf + nb)]
    for e in ev:
        e.record()
    torch.cuda.synchronize()
    try:
        m.moe_profile_events(ev)
        layer.backward(x, dout)
    finally:
        m.moe_profile_events(None)
    torch.cuda.synchronize()
    layer.check()
    stages = [ev[nf + i].elapsed_time(ev[nf + i + 1]) for i in range(nb - 1)]
    assert len(stages) == len(m.PROFILE_BWD_STAGES)
    assert all(t >= 0.0 for t in stages), stages
    total = ev[nf].elapsed_time(ev[nf + nb - 1])
    assert abs(sum(stages) - total) <= 1e-3 * max(total, 1e-3) + 1e-3
