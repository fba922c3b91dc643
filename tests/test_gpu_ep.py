"""GPU parity of the expert-parallel layer's kernels (dispatch packing, the
experts over received packed rows, combine), with W ranks' work run in one
process on one GPU (sparse_moe_layer_expert_b200.ep.forward_local: the
exchanges are copies between the ranks' buffers).  Each rank's output is
compared with the oracle's single-device layer for its tokens, and the
dispatch bookkeeping with the oracle's dispatch plan on the GPU's own routing
("DeepSeek-V3 Technischer Bericht", Methode section 2; the all-to-all
dispatch/combine of "Problem und Motivation" item 2)."""
import numpy as np
import pytest
import torch

import moe_synth as S
from _moe_util import NEAR_TIE, Problem, assert_close, bf16_to_f64, oracle_cfg, shape_of
from test_gpu_layer import build_gpu_layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def m():
    import sparse_moe_layer_expert_b200 as pkg
    return pkg


def _experts(oracle_lib, prob):
    return [prob.oracle_expert(oracle_lib, e) for e in range(prob.E)]


@pytest.mark.parametrize("W,groups", [(1, 0), (2, 0), (4, 0), (4, 4)])
def test_ep_layer_matches_oracle(m, oracle_lib, W, groups):
    from sparse_moe_layer_expert_b200.ep import LibraryOps, forward_local
    from oracle.ep import dispatch_plan
    cfg = dict(S.TINY, n_groups=groups, topk_groups=2 if groups else 0)
    prob = Problem(cfg, 8, seed=80 + W + groups)
    layer = build_gpu_layer(m, prob)
    ops = [LibraryOps(layer, W, r) for r in range(W)]
    xs = [S.gen_x(64 + 37 * r, cfg["H"], 90 + 7 * r + W).cuda() for r in range(W)]  # ragged per rank
    outs = forward_local(ops, xs, m.MOE_DTYPE_F32)
    layer.check()
    ocf = oracle_cfg(oracle_lib, cfg)
    experts = _experts(oracle_lib, prob)
    for r in range(W):
        x = xs[r].cpu()
        # the dispatch bookkeeping, exactly, on the GPU's own routing
        xq, xsc, idx, gate = ops[r].quant_route(xs[r])
        send, counts, row_of, _ = ops[r].dispatch(xq, xsc, idx, gate)
        plans = dispatch_plan(idx.cpu().numpy(), gate.cpu().numpy(), cfg["Nr"], W)
        assert counts == [len(p[0]) for p in plans]
        ro = row_of.cpu().numpy()
        base = 0
        for d, (toks, slots, gates) in enumerate(plans):
            assert (ro[toks, d] == base + np.arange(len(toks))).all()
            assert (np.delete(ro[:, d], toks) == -1).all()
            rows = send[base:base + len(toks)].cpu().numpy()
            H, Kr = cfg["H"], cfg["Kr"]
            assert np.array_equal(rows[:, :H], xq.cpu().numpy()[toks])
            o = H + 4 * (H // 128)
            got_slots = np.ascontiguousarray(rows[:, o:o + 4 * Kr]).view(np.int32)
            got_gates = np.ascontiguousarray(rows[:, o + 4 * Kr:o + 8 * Kr]).view(np.float32)
            assert np.array_equal(got_slots, slots)
            assert np.array_equal(got_gates, gates.astype(np.float32))
            base += len(toks)
        # the output against the single-device oracle (tokens off near-ties)
        res = oracle_lib.forward(ocf, x, prob.wr, prob.bias, experts)
        keep = res["gap"] >= NEAR_TIE
        got = outs[r].cpu().numpy().astype(np.float64)[keep]
        assert_close(got, res["out"][keep], what=f"expert-parallel output, rank {r} of {W}")
        # and against the single-device library layer on the same tokens
        one = layer.forward(xs[r], out_dtype=m.MOE_DTYPE_F32)
        assert_close(got, one.cpu().numpy().astype(np.float64)[keep], what="vs single-device layer")


def test_ep_experts_rejects_bad_rows(m):
    prob = Problem(S.TINY, 8, seed=3)
    layer = build_gpu_layer(m, prob)
    from sparse_moe_layer_expert_b200.ep import LibraryOps
    ops = LibraryOps(layer, 2, 0)
    rows = torch.zeros((4, ops.row_bytes + 16), dtype=torch.uint8, device="cuda")
    with pytest.raises(m.MoeError) as e:
        m.moe_ep_experts(ops.cfg_local, ops.w_local, rows, torch.empty((4, 512), dtype=torch.bfloat16, device="cuda"))
    assert e.value.status == m.MOE_ERR_INVALID_ARG
