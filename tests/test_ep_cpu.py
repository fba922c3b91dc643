"""Expert-parallel bookkeeping on CPU: two gloo ranks run the package's
expert-parallel layer (sparse_moe_layer_expert_b200.ep: dispatch counts,
the row exchange to the experts' ranks, the reverse exchange of the partial
sums, the combine) with the device steps replaced by the oracle's double-
precision routines working on the same packed-row layout the library uses.
Each rank's output must equal the single-device layer oracle's for its own
tokens ("DeepSeek-V3 Technischer Bericht", Methode section 2; the exchange is
the pages' all-to-all dispatch/combine, "Problem und Motivation" item 2).
"""
import json
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SHAPE = dict(H=256, I=128, Nr=8, Kr=3, Ns=1)


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _bf16_round(v: np.ndarray) -> np.ndarray:
    """Round doubles to bf16 (through the oracle) and back to doubles."""
    import oracle
    bits = oracle.round_bf16(v).astype(np.uint32) << 16
    return bits.view(np.float32).astype(np.float64)


class OracleOps:
    """The device steps of one rank, computed by the oracle on the host, in
    the library's packed-row layout: codes, scales, int32 local expert per
    slot (-1 elsewhere), FP32 gate per slot, padded to 16 bytes."""

    def __init__(self, world, rank, seed):
        import oracle
        import moe_synth as S
        H, I, Nr, Kr = SHAPE["H"], SHAPE["I"], SHAPE["Nr"], SHAPE["Kr"]
        self.world, self.rank = world, rank
        self.cf = oracle.cfg(H, I, Nr, Kr)
        self.wr = S.gen_router(Nr, H, seed)
        self.bias = S.gen_bias(Nr, seed)
        self.expert_w = []
        for e in range(Nr + 1):
            w13, w2 = S.gen_expert(e, H, I, seed)
            a, sa = oracle.quant_128x128(w13)
            b, sb = oracle.quant_128x128(w2)
            self.expert_w.append((a, sa, b, sb))
        self.per = Nr // world
        self.row_bytes = (H + 4 * (H // 128) + 8 * Kr + 15) // 16 * 16

    def _pack(self, xq, xs, slots, gates):
        H, Kr = SHAPE["H"], SHAPE["Kr"]
        n = xq.shape[0]
        rows = np.zeros((n, self.row_bytes), np.uint8)
        rows[:, :H] = xq
        rows[:, H:H + 4 * (H // 128)] = np.ascontiguousarray(xs, np.float32).view(np.uint8).reshape(n, -1)
        o = H + 4 * (H // 128)
        rows[:, o:o + 4 * Kr] = np.ascontiguousarray(slots, np.int32).view(np.uint8).reshape(n, -1)
        rows[:, o + 4 * Kr:o + 8 * Kr] = np.ascontiguousarray(gates, np.float32).view(np.uint8).reshape(n, -1)
        return rows

    def _unpack(self, rows):
        H, Kr = SHAPE["H"], SHAPE["Kr"]
        n = rows.shape[0]
        o = H + 4 * (H // 128)
        xq = np.ascontiguousarray(rows[:, :H])
        xs = np.ascontiguousarray(rows[:, H:o]).view(np.float32).reshape(n, -1)
        slots = np.ascontiguousarray(rows[:, o:o + 4 * Kr]).view(np.int32).reshape(n, Kr)
        gates = np.ascontiguousarray(rows[:, o + 4 * Kr:o + 8 * Kr]).view(np.float32).reshape(n, Kr)
        return xq, xs, slots, gates

    def quant_route(self, x):
        import oracle
        xq, xs = oracle.quant_1x128(x)
        idx, gate, _, _ = oracle.route(self.cf, x, self.wr, self.bias)
        return xq, xs, idx, gate

    def dispatch(self, xq, xs, idx, gate):
        from oracle.ep import dispatch_plan
        T, W, Kr = xq.shape[0], self.world, SHAPE["Kr"]
        plans = dispatch_plan(idx, gate, SHAPE["Nr"], W)
        row_of = np.full((T, W), -1, np.int32)
        blocks, counts, r = [], [], 0
        for d, (toks, slots, gates) in enumerate(plans):
            blocks.append(self._pack(xq[toks], xs[toks], slots, gates.astype(np.float32)))
            row_of[toks, d] = r + np.arange(len(toks))
            counts.append(len(toks))
            r += len(toks)
        send = torch.from_numpy(np.concatenate(blocks, axis=0))
        sl = np.full((T, Kr), -1, np.int32)
        sl[:, 0] = 0
        gs = np.zeros((T, Kr), np.float32)
        gs[:, 0] = 1.0
        self_rows = self._pack(xq, xs, sl, gs)
        return send, counts, row_of, self_rows

    def _run(self, rows, experts_local):
        import oracle
        xq, xs, slots, gates = self._unpack(np.asarray(rows))
        out = np.zeros((xq.shape[0], SHAPE["H"]), np.float64)
        for i in range(xq.shape[0]):
            for k in range(SHAPE["Kr"]):
                j = int(slots[i, k])
                if j >= 0:
                    out[i] += float(gates[i, k]) * oracle.expert_ffn(self.cf, xq[i:i + 1], xs[i:i + 1],
                                                                     *experts_local[j])[0]
        # the partial sums travel as bf16, as the library's do
        return torch.from_numpy(_bf16_round(out))

    def experts(self, rows):
        loc = self.expert_w[self.rank * self.per:(self.rank + 1) * self.per]
        return self._run(rows.numpy(), loc)

    def shared(self, self_rows):
        return self._run(self_rows, [self.expert_w[SHAPE["Nr"]]])

    def combine(self, x, row_of, back, y_shared, out_dtype=None):
        u = x.float().numpy().astype(np.float64)
        out = u + y_shared.numpy()
        b = back.numpy()
        for t in range(u.shape[0]):
            for d in range(self.world):
                if row_of[t, d] >= 0:
                    out[t] += b[row_of[t, d]]
        return out


def _rank_main(rank: int, world: int, port: int, out_dir: str):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import datetime

    import torch.distributed as dist

    import moe_synth as S
    import oracle
    from sparse_moe_layer_expert_b200.ep import EpMoeLayer, TorchExchange
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        seed = 5
        ops = OracleOps(world, rank, seed)
        x = S.gen_x(20 + 7 * rank, SHAPE["H"], 100 + rank)  # ragged token counts per rank
        layer = EpMoeLayer(ops, TorchExchange())
        out = layer.forward(x)
        ref = oracle.forward(ops.cf, x, ops.wr, ops.bias, ops.expert_w)["out"]
        err = float(np.abs(out - ref).max())
        rms = float(np.sqrt(np.mean(ref ** 2)))
        rel = float(np.linalg.norm(out - ref) / np.linalg.norm(ref))
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump(dict(rank=rank, err=err, rms=rms, rel=rel, T=int(x.shape[0])), f)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_expert_parallel_layer_on_gloo_ranks(tmp_path, world):
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, str(tmp_path))) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
    for p in procs:
        if p.is_alive():
            p.kill()
            pytest.fail("a rank did not finish")
        assert p.exitcode == 0
    for r in range(world):
        d = json.load(open(tmp_path / f"rank{r}.json"))
        # the partial sums and the shared expert's output travel as bf16:
        # within the layer's tolerance (rel-Frobenius 2e-3, max 1e-2 rms)
        assert d["rel"] <= 2e-3 and d["err"] <= 1e-2 * d["rms"], d


def test_local_exchange_routes_blocks_to_their_ranks():
    sys.path.insert(0, ROOT)
    from sparse_moe_layer_expert_b200.ep import LocalExchange
    W = 3
    # rank s sends rows tagged (s, d, i) to d
    counts = [[1, 0, 2], [2, 1, 0], [0, 3, 1]]
    sends = []
    for s in range(W):
        rows = [[s, d, i] for d in range(W) for i in range(counts[s][d])]
        sends.append(torch.tensor(rows, dtype=torch.int64).reshape(-1, 3))
    recv = LocalExchange.rows(sends, counts)
    for d in range(W):
        want = [[s, d, i] for s in range(W) for i in range(counts[s][d])]
        assert recv[d].tolist() == want
    assert LocalExchange.counts(counts) == [[1, 2, 0], [0, 1, 3], [2, 0, 1]]
