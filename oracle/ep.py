"""Expert-parallel decomposition of the layer -- TEST INFRASTRUCTURE ONLY.

The DeepSeek-V3 pages place the routed experts of a layer on different GPUs
and move tokens to them and back with all-to-all exchanges ("DeepSeek-V3
Technischer Bericht" (xyznot.com/de), "Problem und Motivation" item 2 and
"Kernideen", DualPipe bullet: all-to-all dispatch and combine of the MoE
layer; "DeepSeek-V3 技術報告書" (singularity-lens.com), DualPipe paragraph:
dispatch/combine communication).  They fix no data layout; this module
writes out the plainest one, in the layer's own terms, so that the
distributed path can be checked against the single-device layer:

  * W ranks; rank d owns the routed experts [d*N_r/W, (d+1)*N_r/W);
    every rank holds the router, the shared expert and its own tokens;
  * dispatch r -> d: the tokens of rank r that selected at least one expert
    of rank d, in token order, each sent once (its FP8 row and 1x128 scales),
    with the list of its slots k whose expert lives on d (expert, gate);
  * rank d receives the rows of ranks 0..W-1 in rank order, applies, per row,
    each listed expert to the row, scales by the gate and adds the results in
    slot order: one partial sum per received row;
  * combine at r: out_t = u_t + FFN_shared(u_t) + sum over d ascending of the
    partial that rank d returned for token t.

Mathematically the result is the layer's h'_t ("DeepSeek-V3 Technischer
Bericht", Methode section 2): the same terms, added in another order.  The
functions here compute in double precision through the oracle's own C
routines and share nothing with the CUDA library.
"""
from __future__ import annotations

import numpy as np

from . import _u16, expert_ffn, quant_1x128, route


def owner(e: int, Nr: int, W: int) -> int:
    """Rank that owns routed expert e (contiguous equal blocks)."""
    return int(e) // (Nr // W)


def dispatch_plan(idx: np.ndarray, gate: np.ndarray, Nr: int, W: int):
    """For one rank's routing decision (idx, gate [T, K_r]) the rows it sends
    to each destination.  Returns a list over d of (tokens [n_d], slots
    [n_d, K_r] local expert id or -1, gates [n_d, K_r] (0 where unused)).
    A token appears at most once per destination, in token order."""
    idx = np.asarray(idx)
    T, Kr = idx.shape
    per = Nr // W
    plans = []
    for d in range(W):
        toks, slots, gates = [], [], []
        for t in range(T):
            row_s = np.full(Kr, -1, np.int32)
            row_g = np.zeros(Kr, np.float64)
            hit = False
            for k in range(Kr):
                e = int(idx[t, k])
                if e // per == d:
                    row_s[k] = e - d * per
                    row_g[k] = gate[t, k]
                    hit = True
            if hit:
                toks.append(t)
                slots.append(row_s)
                gates.append(row_g)
        plans.append((np.array(toks, np.int64), np.array(slots, np.int32).reshape(-1, Kr),
                      np.array(gates, np.float64).reshape(-1, Kr)))
    return plans


def expert_side(cf, xq_rows, xs_rows, slots, gates, experts_local):
    """Rank d's work: for every received row, sum over its listed slots (in
    slot order) of gate * FFN_e(row).  experts_local[j] = (W13q, s13, W2q,
    s2) of the rank's j-th expert.  Returns partial sums [n, H] (double)."""
    n = xq_rows.shape[0]
    out = np.zeros((n, cf.H), np.float64)
    for i in range(n):
        for k in range(slots.shape[1]):
            j = int(slots[i, k])
            if j < 0:
                continue
            y = expert_ffn(cf, xq_rows[i:i + 1], xs_rows[i:i + 1], *experts_local[j])
            out[i] += gates[i, k] * y[0]
    return out


def forward_ep(cf, xs_by_rank, Wr, bias, experts, W: int):
    """The layer over W ranks' token sets by dispatch, expert-side partial
    sums and combine.  xs_by_rank: list of bf16 [T_r, H] inputs; experts: the
    N_r + N_s expert tuples (routed first, then shared).  Returns (outputs per
    rank [T_r, H] double, the send counts [W, W] of rows r -> d)."""
    Nr, Ns = cf.Nr, cf.Ns
    per = Nr // W
    assert Nr % W == 0
    routed = []
    quant = []
    for x in xs_by_rank:
        idx, gate, _, _ = route(cf, x, Wr, bias)
        routed.append((idx, gate))
        quant.append(quant_1x128(x, cf.scale_mode))
    plans = [dispatch_plan(idx, gate, Nr, W) for idx, gate in routed]
    counts = np.array([[len(plans[r][d][0]) for d in range(W)] for r in range(W)], np.int64)
    # expert side: rank d processes what every rank r sent it, in rank order
    partial = {}
    for d in range(W):
        loc = [experts[d * per + j] for j in range(per)]
        for r in range(W):
            toks, slots, gates = plans[r][d]
            if len(toks) == 0:
                continue
            xq, xs = quant[r]
            partial[(r, d)] = expert_side(cf, xq[toks], xs[toks], slots, gates, loc)
    # combine at the source rank: residual, shared expert(s), then the
    # partials of the destinations in ascending rank order
    outs = []
    for r, x in enumerate(xs_by_rank):
        xq, xs = quant[r]
        bits = _u16(x).astype(np.uint32) << 16  # bf16 -> float32 bit pattern
        o = bits.view(np.float32).astype(np.float64)
        for e in range(Nr, Nr + Ns):
            o += expert_ffn(cf, xq, xs, *experts[e])
        for d in range(W):
            toks = plans[r][d][0]
            if len(toks):
                o[toks] += partial[(r, d)]
        outs.append(o)
    return outs, counts
