"""Expert-parallel DeepSeekMoE layer: one rank per GPU, routed experts split
over the ranks, tokens exchanged by all-to-all ("DeepSeek-V3 Technischer
Bericht", "Problem und Motivation" item 2 and "Kernideen", DualPipe bullet).

Plumbing only.  Every step that touches the layer's numbers runs in
libmoefp8's kernels (quantize, route, dispatch packing, the grouped expert
GEMMs, combine); this module sizes the buffers, moves the packed rows between
ranks and keeps the bookkeeping of which rows went where:

  1. each rank quantizes and routes its own tokens;
  2. dispatch: one packed row per (token, destination rank owning one of its
     experts), grouped by destination; the per-destination counts are
     exchanged first so every rank knows how many rows it will receive;
  3. rows r -> d (all-to-all); rank d runs its experts on what it received
     and gets one gate-weighted partial sum (bf16) per received row;
  4. the partial sums go back d -> r (the reverse all-to-all) into the send
     buffer's row order; the shared expert runs on the rank's own tokens;
  5. combine: u_t + shared + the returned partial sums.

The exchange is a pluggable object: `TorchExchange` uses torch.distributed
(NCCL over NVLink on GPUs, gloo on CPUs), `LocalExchange` passes buffers
between ranks held in one process (several ranks' worth of work on one
device, with no waiting between them).  The device steps are a pluggable
`ops` object too: `LibraryOps` calls the library.
"""
from __future__ import annotations

import torch

from . import _binding as B


# ------------------------------------------------------------------ device steps
class LibraryOps:
    """The device steps of one rank, in libmoefp8's kernels."""

    def __init__(self, layer, world: int, rank: int):
        """layer: a MoeLayer holding the whole layer's weights (routed experts
        0..N_r-1, then the shared expert); this rank keeps views of its own
        experts' slices and of the shared expert."""
        c = layer.cfg
        assert c.n_routed % world == 0 and c.n_shared == 1
        self.layer, self.world, self.rank = layer, world, rank
        self.cfg = c
        per = c.n_routed // world
        sl = slice(rank * per, (rank + 1) * per)
        self.w_local = dict(w13=layer.w13[sl], s13=layer.s13[sl], w2=layer.w2[sl], s2=layer.s2[sl])
        sh = slice(c.n_routed, c.n_routed + 1)
        self.w_shared = dict(w13=layer.w13[sh], s13=layer.s13[sh], w2=layer.w2[sh], s2=layer.s2[sh])
        base = dict(layer.shape, Ns=0, n_groups=0, topk_groups=0)
        self.cfg_local = B.config_from(dict(base, Nr=per))
        self.cfg_shared = B.config_from(dict(base, Nr=1))
        self.row_bytes = B.moe_ep_row_bytes(c)
        self.device = layer.device
        self.err = layer.err

    def quant_route(self, x):
        pow2 = self.cfg.scale_mode == B.MOE_SCALE_POW2
        xq, xs = B.fp8_quant_1x128(x, pow2=pow2)
        idx, gate, _ = B.moe_route(self.cfg, x, self.layer.wr, self.layer.bias, err=self.err)
        return xq, xs, idx, gate

    def dispatch(self, xq, xs, idx, gate):
        T, W, Kr = xq.shape[0], self.world, self.cfg.top_k
        dev = self.device
        cap = T * min(W, Kr)
        send = torch.empty((cap, self.row_bytes), dtype=torch.uint8, device=dev)
        counts = torch.empty(W, dtype=torch.int32, device=dev)
        offsets = torch.empty(W + 1, dtype=torch.int32, device=dev)
        row_of = torch.empty((T, W), dtype=torch.int32, device=dev)
        self_rows = torch.empty((T, self.row_bytes), dtype=torch.uint8, device=dev)
        B.moe_ep_dispatch(self.cfg, W, xq, xs, idx, gate, send, counts, offsets, row_of, self_rows, err=self.err)
        return send, counts.cpu().tolist(), row_of, self_rows

    def experts(self, rows):
        out = torch.empty((rows.shape[0], self.cfg.hidden), dtype=torch.bfloat16, device=self.device)
        return B.moe_ep_experts(self.cfg_local, self.w_local, rows, out, err=self.err)

    def shared(self, self_rows):
        out = torch.empty((self_rows.shape[0], self.cfg.hidden), dtype=torch.bfloat16, device=self.device)
        return B.moe_ep_experts(self.cfg_shared, self.w_shared, self_rows, out, err=self.err)

    def combine(self, x, row_of, back, y_shared, out_dtype=B.MOE_DTYPE_BF16):
        dt = torch.float32 if out_dtype == B.MOE_DTYPE_F32 else torch.bfloat16
        out = torch.empty(x.shape, dtype=dt, device=self.device)
        return B.moe_ep_combine(self.cfg, self.world, x, row_of, back, y_shared, out, out_dtype)


# -------------------------------------------------------------------- exchanges
def _rows_by_source(buf, counts):
    """Split a row buffer into consecutive blocks of counts[i] rows."""
    out, r = [], 0
    for c in counts:
        out.append(buf[r:r + c])
        r += c
    return out


class TorchExchange:
    """All-to-all exchanges of one rank through torch.distributed."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group

    def counts(self, send_counts):
        W = len(send_counts)
        s = torch.tensor(send_counts, dtype=torch.int64)
        if self.dist.get_backend(self.group) == "nccl":
            s = s.cuda()
        r = torch.empty_like(s)
        self.dist.all_to_all_single(r, s, group=self.group)
        out = r.cpu().tolist()
        assert len(out) == W
        return out

    def rows(self, send, send_counts, recv_counts):
        """Rows of send (grouped by destination, send_counts each) to their
        destinations; returns the received rows grouped by source."""
        width = send.shape[1]
        flat = send[:sum(send_counts)].contiguous().view(torch.uint8).reshape(-1)
        recv = torch.empty((sum(recv_counts), width), dtype=send.dtype, device=send.device)
        self.dist.all_to_all_single(recv.view(torch.uint8).reshape(-1), flat,
                                    [c * width * send.element_size() for c in recv_counts],
                                    [c * width * send.element_size() for c in send_counts], group=self.group)
        return recv


class LocalExchange:
    """Exchanges between the ranks of one process (each list index is a
    rank): what rank r sends to d is the d-th block of its send buffer."""

    @staticmethod
    def counts(all_send_counts):
        W = len(all_send_counts)
        return [[all_send_counts[s][d] for s in range(W)] for d in range(W)]

    @staticmethod
    def rows(all_send, all_send_counts):
        W = len(all_send)
        blocks = [_rows_by_source(all_send[s], all_send_counts[s]) for s in range(W)]
        return [torch.cat([blocks[s][d] for s in range(W)], dim=0) for d in range(W)]


# ------------------------------------------------------------------ the layer
class EpMoeLayer:
    """One rank of the expert-parallel layer (forward)."""

    def __init__(self, ops, exchange):
        self.ops = ops
        self.ex = exchange

    def forward(self, x, out_dtype=B.MOE_DTYPE_BF16):
        ops = self.ops
        xq, xs, idx, gate = ops.quant_route(x)
        send, send_counts, row_of, self_rows = ops.dispatch(xq, xs, idx, gate)
        recv_counts = self.ex.counts(send_counts)
        recv = self.ex.rows(send, send_counts, recv_counts)
        partial = ops.experts(recv)
        # the partial sums go back: rank d returns to s the rows s sent it,
        # in the order s sent them, so they land in s's send-buffer order
        back = self.ex.rows(partial, recv_counts, send_counts)
        y_sh = ops.shared(self_rows)
        return ops.combine(x, row_of, back, y_sh, out_dtype)


def forward_local(ops_by_rank, xs, out_dtype=B.MOE_DTYPE_BF16):
    """The expert-parallel forward of W ranks held in one process, step by
    step across the ranks (each rank's kernels run on its own buffers; the
    exchanges are copies between them).  Returns the outputs per rank."""
    W = len(ops_by_rank)
    st = [ops.quant_route(x) for ops, x in zip(ops_by_rank, xs)]
    disp = [ops.dispatch(*s) for ops, s in zip(ops_by_rank, st)]
    send_counts = [d[1] for d in disp]
    recv = LocalExchange.rows([d[0] for d in disp], send_counts)
    partial = [ops_by_rank[d].experts(recv[d]) for d in range(W)]
    recv_counts = LocalExchange.counts(send_counts)
    back = LocalExchange.rows(partial, recv_counts)
    outs = []
    for r in range(W):
        y_sh = ops_by_rank[r].shared(disp[r][3])
        outs.append(ops_by_rank[r].combine(xs[r], disp[r][2], back[r], y_sh, out_dtype))
    return outs
