"""Pins of the oracle's expert-parallel decomposition (oracle/ep.py): the
dispatch plan against hand-worked values and its invariants, and the
distributed layer (dispatch, expert-side partial sums, combine) against the
single-device layer oracle -- the same terms of h'_t ("DeepSeek-V3
Technischer Bericht", Methode section 2) added in another order, so they
agree to double-precision rounding."""
import numpy as np
import pytest

import moe_synth as S


def test_dispatch_plan_hand_worked():
    from oracle.ep import dispatch_plan
    # 3 tokens, K_r = 2, 8 experts on 2 ranks (experts 0..3 on rank 0)
    idx = np.array([[1, 5], [6, 7], [0, 3]], np.int32)
    gate = np.array([[0.6, 0.4], [0.7, 0.3], [0.2, 0.8]])
    p0, p1 = dispatch_plan(idx, gate, 8, 2)
    assert p0[0].tolist() == [0, 2]                       # token 1 sends nothing to rank 0
    assert p0[1].tolist() == [[1, -1], [0, 3]]            # local expert ids per slot
    assert np.allclose(p0[2], [[0.6, 0.0], [0.2, 0.8]])
    assert p1[0].tolist() == [0, 1]                       # token 1 once, although both slots go there
    assert p1[1].tolist() == [[-1, 1], [2, 3]]
    assert np.allclose(p1[2], [[0.0, 0.4], [0.7, 0.3]])


@pytest.mark.parametrize("W", [1, 2, 4, 8])
def test_dispatch_plan_invariants(W):
    from oracle.ep import dispatch_plan
    rng = np.random.default_rng(W)
    T, Kr, Nr = 50, 4, 16
    idx = np.stack([rng.choice(Nr, Kr, replace=False) for _ in range(T)]).astype(np.int32)
    gate = rng.random((T, Kr))
    plans = dispatch_plan(idx, gate, Nr, W)
    used = 0
    for d, (toks, slots, gates) in enumerate(plans):
        assert len(set(toks.tolist())) == len(toks) and list(toks) == sorted(toks)   # once, in token order
        for t, srow, grow in zip(toks, slots, gates):
            for k in range(Kr):
                e = idx[t, k]
                if e // (Nr // W) == d:
                    assert srow[k] == e - d * (Nr // W) and grow[k] == gate[t, k]
                else:
                    assert srow[k] == -1 and grow[k] == 0.0
        used += int((slots >= 0).sum())
    assert used == T * Kr                                                            # every assignment once
    # a token reaches exactly the ranks that own one of its experts
    for t in range(T):
        dests = {d for d, (toks, _, _) in enumerate(plans) if t in set(toks.tolist())}
        assert dests == {int(e) // (Nr // W) for e in idx[t]}


@pytest.mark.parametrize("W,groups", [(1, 0), (2, 0), (4, 0), (4, 4)])
def test_forward_ep_equals_single_device_layer(oracle_lib, W, groups):
    from oracle.ep import forward_ep
    H, I, Nr, Kr = 256, 128, 16, 4
    cf = oracle_lib.cfg(H, I, Nr, Kr, 1, groups, 2 if groups else 0)
    seed = 70 + W + groups
    xs = [S.gen_x(24 + 5 * r, H, seed + r) for r in range(W)]   # ragged token counts per rank
    wr = S.gen_router(Nr, H, seed)
    bias = S.gen_bias(Nr, seed)
    experts = []
    for e in range(Nr + 1):
        w13, w2 = S.gen_expert(e, H, I, seed)
        a, sa = oracle_lib.quant_128x128(w13)
        b, sb = oracle_lib.quant_128x128(w2)
        experts.append((a, sa, b, sb))
    outs, counts = forward_ep(cf, xs, wr, bias, experts, W)
    for r, x in enumerate(xs):
        ref = oracle_lib.forward(cf, x, wr, bias, experts)["out"]
        assert np.allclose(outs[r], ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    # rows sent: each token once per destination that owns one of its experts
    assert counts.shape == (W, W)
    assert (counts.sum(axis=1) <= np.array([x.shape[0] * Kr for x in xs])).all()
    if groups == W:
        # groups of experts coincide with ranks: a token reaches at most
        # topk_groups ranks
        assert (counts.sum(axis=1) <= np.array([x.shape[0] * 2 for x in xs])).all()
