"""GPU parity of the FP8 backward of the expert FFNs (moe_backward, routing
held fixed) against the oracle's layer backward (oracle/backward.py): the
input gradient dx and every expert's weight gradients dW13, dW2, on the small
configuration (all tokens; experts with several 128-token tiles and ragged
tails) and on one expert at full DeepSeek-V3 size ("DeepSeek-V3 Technischer
Bericht", Kernideen, FP8 bullet: E4M3 for all tensors; the backward tile
orientation is the reading the oracle documents).  Tolerance: the layer's
stated bound (relative Frobenius error 2e-3, max |diff| 1e-2 rms) on every
FP32 output."""
import numpy as np
import pytest
import torch

import moe_synth as S
from _moe_util import NEAR_TIE, Problem, assert_close, oracle_cfg
from test_gpu_layer import build_gpu_layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def m():
    import sparse_moe_layer_expert_b200 as pkg
    return pkg


def run_backward_case(m, oracle_lib, cfg, T, seed, bias_shift=None, tokens_checked=None):
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
    dx, dW13, dW2 = layer.backward(x, dout.cuda())
    layer.check()
    experts = [prob.oracle_expert(oracle_lib, e) for e in range(prob.E)]
    ocf = oracle_cfg(oracle_lib, cfg)
    ref = OB.layer_backward(ocf, prob.x, prob.wr, prob.bias, experts, dout)
    # the same routing on both sides (the configurations are chosen without near-ties)
    assert (ref["gap"] >= NEAR_TIE).all()
    got_idx = idx_out.cpu().numpy()
    for t in range(T):
        assert set(got_idx[t].tolist()) == set(ref["idx"][t].tolist()), t
    H, I, Kr, Ns = cfg["H"], cfg["I"], cfg["Kr"], cfg.get("Ns", 1)
    R, E = T * Kr, prob.E
    RS = R + T * Ns
    # the backward's own intermediates, step by step against the oracle's
    # expert backward on the same tokens
    bws, BL = layer.backward_workspace(T), m.moe_backward_workspace_layout(layer.cfg, T)

    def view(name, shape):
        off, nb = BL[name]
        n = int(np.prod(shape))
        assert n * 4 <= nb
        return bws[off:off + 4 * n].view(torch.float32).view(shape).cpu().numpy().astype(np.float64)

    GU, dh, hh, dGU = view("gu", (RS, 2 * I)), view("dh", (RS, I)), view("h", (RS, I)), view("dgu", (RS, 2 * I))
    ws, L = layer.workspace(T), layer.layout(T)
    offsets = m.ws_view(ws, L, "offsets", torch.int32, (cfg["Nr"] + 1,)).cpu().numpy()
    xu = prob.x
    d32 = dout.float().numpy()
    msgs, fails = [], []
    for e in sorted(ref["dW13"].keys()):
        if e < cfg["Nr"]:
            toks, slots = np.nonzero(ref["idx"] == e)
            order = np.argsort(toks, kind="stable")
            toks, slots = toks[order], slots[order]
            rows = np.arange(offsets[e], offsets[e + 1])
            dy = (ref["gate"][toks, slots].astype(np.float32)[:, None] * d32[toks]).astype(np.float32)
        else:
            toks = np.arange(T)
            rows = R + toks
            dy = d32
        r = OB.expert_backward(xu[torch.as_tensor(toks)], dy, *experts[e])
        for nm, got, want in (("G", GU[rows, :I], r["G"]), ("U", GU[rows, I:], r["U"]), ("dh", dh[rows], r["dh"]),
                              ("h", hh[rows], r["h"]), ("dG", dGU[rows, :I], r["dG"]),
                              ("dU", dGU[rows, I:], r["dU"])):
            rel = np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30)
            msgs.append(f"expert {e} {nm}: rel-Frobenius {rel:.2e}")
            if not rel < 1e-4:
                fails.append(msgs[-1])
        # the weight-gradient GEMM on the GPU's own operands (its dY, h, dG|dU
        # and x), quantized 128x1 by the oracle: only the GEMM's FP32 rounding
        # separates the two
        dyq, dys = OB.quant_128x1_f32(dy)
        hq, hs = OB.quant_128x1_f32(hh[rows].astype(np.float32))
        w2_own = OB.rows_scaled_gemm(dyq.T, dys.T, hq.T, hs.T)
        gq, gs = OB.quant_128x1_f32(dGU[rows].astype(np.float32))
        xq, xs = OB.quant_128x1_bf16(xu[torch.as_tensor(toks)])
        w13_own = OB.rows_scaled_gemm(gq.T, gs.T, xq.T, xs.T)
        got13, got2 = dW13[e].cpu().numpy().astype(np.float64), dW2[e].cpu().numpy().astype(np.float64)
        for nm, got, want in (("dW13 (own operands)", got13, w13_own), ("dW2 (own operands)", got2, w2_own)):
            rel = np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30)
            msgs.append(f"expert {e} {nm}: rel-Frobenius {rel:.2e}")
            if not rel < 1e-5:
                fails.append(msgs[-1])
    print("\n".join(msgs[:60]))
    assert not fails, fails[:10]
    dx_h = dx.cpu().numpy().astype(np.float64)
    assert_close(dx_h, ref["dx"], what="dx")
    dW13_h, dW2_h = dW13.cpu().numpy(), dW2.cpu().numpy()
    used = set(ref["dW13"].keys())
    for e in range(E):
        if e in used:
            assert_close(dW13_h[e].astype(np.float64), ref["dW13"][e], what=f"dW13 of expert {e}")
            assert_close(dW2_h[e].astype(np.float64), ref["dW2"][e], what=f"dW2 of expert {e}")
        else:
            assert not dW13_h[e].any() and not dW2_h[e].any(), f"expert {e} has no token but a gradient"
    return ref


def test_backward_tiny(m, oracle_lib):
    run_backward_case(m, oracle_lib, dict(S.TINY), 256, 0)


def test_backward_tiny_multi_tile_experts(m, oracle_lib):
    # every token picks experts 0..K_r-1: each holds T = 300 rows, three
    # 128-token tiles of the weight gradients (the last one 44 rows)
    ref = run_backward_case(m, oracle_lib, dict(S.TINY), 300, 3, bias_shift=S.TINY["Kr"])
    assert set(ref["dW13"].keys()) == set(range(S.TINY["Kr"])) | {S.TINY["Nr"]}


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
