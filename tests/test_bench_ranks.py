"""Multi-rank host logic of bench.py, on CPU with the gloo backend (world size 2).

bench.py runs one process per GPU; the timed region's length is the maximum over
ranks and the value is the whole job's tokens/s.  These tests run the same
helpers in two gloo processes on the host, with no GPU and no CUDA library.
"""
import json
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out_dir: str):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import datetime

    import torch.distributed as dist

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        r, w, local = bench.dist_env()
        # each rank's own timed region (ms over 10 steps); rank 1 is the slower one
        mine = 40.0 + 10.0 * rank
        bench.barrier(w)
        total = bench.max_over_ranks(mine, w)
        ms_per_step, value = bench.aggregate(total, 10, w, 4096)
        # the reference arm: only rank 0 works, the others return at once with no output
        ref_rc = bench.run_reference(bench.parse(["--impl", "reference"]), r, w) if r != 0 else None
        bench.barrier(w)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump(dict(rank=r, world=w, local=local, total=total, ms_per_step=ms_per_step, value=value,
                           ref_rc=ref_rc), f)
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_rank_and_aggregate_tokens(tmp_path):
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, str(tmp_path))) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    for p in procs:
        if p.is_alive():
            p.kill()
            pytest.fail("a rank did not finish")
        assert p.exitcode == 0
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r, d in enumerate(res):
        assert (d["rank"], d["world"], d["local"]) == (r, world, r)
        assert d["total"] == 50.0                 # the slower rank's region, on every rank
        assert d["ms_per_step"] == pytest.approx(5.0)
        # whole job: 2 ranks x 4096 tokens per 5 ms step
        assert d["value"] == pytest.approx(2 * 4096 / 5e-3)
    assert res[1]["ref_rc"] == 0


def test_single_rank_helpers_are_identities():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    bench.barrier(1)
    ms, v = bench.aggregate(30.0, 10, 1, 64)
    assert ms == pytest.approx(3.0) and v == pytest.approx(64 / 3e-3)
