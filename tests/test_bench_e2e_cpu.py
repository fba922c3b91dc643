"""Host logic of bench.py's end-to-end legs, on CPU with stand-in streams and
events (no GPU, no CUDA library).

The pipelined leg must (a) run its steps in order on the launching stream,
(b) make every step wait for its own input copy and, from the third step on,
for the read-back of the output two steps earlier (the buffer it overwrites),
(c) make every input copy from the third step on wait until the step two
earlier has finished with its buffer, (d) read every step's output back after
that step, and (e) close the timed region only after both copy streams.
The serial leg copies in, steps and copies out in series on one stream.
The stored DRAM traffic of a kernel is reported only for the sources it was
captured on.
"""
import contextlib
import os
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


class _Log:
    def __init__(self):
        self.ops = []
        self.current = None


class _Stream:
    def __init__(self, log, name):
        self.log, self.name = log, name

    def wait_event(self, ev):
        self.log.ops.append((self.name, "wait", ev.tag))

    def wait_stream(self, other):
        self.log.ops.append((self.name, "wait_stream", other.name))


class _Event:
    count = 0

    def __init__(self, log, **kw):
        _Event.count += 1
        self.log, self.tag = log, f"ev{_Event.count}"

    def record(self, stream=None):
        self.log.ops.append((stream.name if stream is not None else self.log.current, "record", self.tag))

    def elapsed_time(self, other):
        return 7.0


@pytest.fixture
def fake_cuda(monkeypatch):
    import bench
    log = _Log()
    names = iter(["h2d", "d2h", "extra1", "extra2"])
    monkeypatch.setattr(torch.cuda, "Stream", lambda dev=None: _Stream(log, next(names)))
    monkeypatch.setattr(torch.cuda, "Event", lambda **kw: _Event(log, **kw))
    monkeypatch.setattr(torch.cuda, "synchronize", lambda dev=None: None)

    @contextlib.contextmanager
    def stream_ctx(s):
        prev, log.current = log.current, s.name
        try:
            yield
        finally:
            log.current = prev

    monkeypatch.setattr(torch.cuda, "stream", stream_ctx)
    return bench, log


def test_pipelined_leg_orders_copies_and_steps(fake_cuda):
    bench, log = fake_cuda
    main = _Stream(log, "main")
    T, H, steps = 4, 8, 5
    x_h = torch.zeros((T, H), dtype=torch.bfloat16)
    out_h = [torch.zeros((T, H), dtype=torch.bfloat16) for _ in range(2)]
    seen = []

    def step_io(x_in, out_buf):
        log.ops.append((log.current, "step", len(seen)))
        seen.append((x_in.data_ptr(), out_buf.data_ptr()))

    ms = bench.e2e_pipelined(step_io, x_h, out_h, main, "cpu", steps, 1)
    assert ms == 7.0
    ops = log.ops
    # (a) steps in order, on the launching stream, alternating two buffer pairs
    step_ops = [o for o in ops if o[1] == "step"]
    assert [o[2] for o in step_ops] == list(range(steps)) and all(o[0] == "main" for o in step_ops)
    assert seen[0] != seen[1] and all(seen[k] == seen[k % 2] for k in range(steps))
    # events in creation order: e0/e1 timing, then x_ready[2], computed[2], read_back[2]
    recs = [(s, t) for s, kind, t in ops if kind == "record"]
    # group each step's records: the h2d stream records x_ready, main records computed, d2h read_back
    x_ready = [t for s, t in recs if s == "h2d"]
    computed = [t for s, t in recs if s == "main"][1:-1]  # drop the timing events e0, e1
    read_back = [t for s, t in recs if s == "d2h"]
    assert len(x_ready) == len(computed) == len(read_back) == steps
    step_idx = [i for i, o in enumerate(ops) if o[1] == "step"]
    for k in range(steps):
        i_step = step_idx[k]
        before = ops[:i_step]
        # (b) the step waits for its input copy and, from k = 2, the read-back two steps earlier
        assert ("main", "wait", x_ready[k]) in before[-3:]
        if k >= 2:
            assert ("main", "wait", read_back[k - 2]) in before[-3:]
            # (c) its input copy waited for step k-2 to finish with the buffer
            rec_x = max(i for i, o in enumerate(ops) if o == ("h2d", "record", x_ready[k]) and i < i_step)
            assert ops[rec_x - 1] == ("h2d", "wait", computed[k - 2])
        # (d) the read-back of step k waits for step k
        i_rb = [i for i, o in enumerate(ops) if o == ("d2h", "record", read_back[k])][-1]
        assert ops[i_rb - 1] == ("d2h", "wait", computed[k]) and i_rb > i_step
    # (e) the end event comes after main waited on both copy streams
    assert ops[-3:] == [("main", "wait_stream", "h2d"), ("main", "wait_stream", "d2h"), ops[-1]]
    assert ops[-1][0] == "main" and ops[-1][1] == "record"
    # the start event precedes every copy: both copy streams wait on it first
    e0 = ops[0]
    assert e0[:2] == ("main", "record") and ops[1:3] == [("h2d", "wait", e0[2]), ("d2h", "wait", e0[2])]


def test_serial_leg_runs_copies_and_steps_in_series(fake_cuda):
    bench, log = fake_cuda
    main = _Stream(log, "main")
    x_h = torch.zeros((4, 8), dtype=torch.bfloat16)
    out_h = torch.zeros((4, 8), dtype=torch.bfloat16)
    calls = []
    ms = bench.e2e_serial(lambda xi, ob: calls.append(log.current), x_h, out_h, main, "cpu", 3, 1)
    assert ms == 7.0 and calls == ["main"] * 3
    assert [o[1] for o in log.ops] == ["record", "record"]


def test_profiled_traffic_is_used_only_for_the_captured_source(tmp_path, monkeypatch):
    import json

    import bench
    k1, k2 = "gemm_fp8_kernel<0>", "gemm_mx_kernel<0>"
    d = {f"{k1}:prefill": dict(bytes_per_launch=123.0, src_sha=bench.gemm_source_sha(k1)),
         f"{k2}:prefill": dict(bytes_per_launch=456.0, src_sha="0" * 16)}
    f = tmp_path / "traffic.json"
    f.write_text(json.dumps(d))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(f))
    assert bench.profiled_traffic("prefill", k1) == 123.0
    assert bench.profiled_traffic("prefill", k2) is None   # captured on other sources
    assert bench.profiled_traffic("decode", k1) is None    # never captured
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "absent.json"))
    assert bench.profiled_traffic("prefill", k1) is None


def test_committed_traffic_figures_match_their_sources():
    """Every DRAM-traffic figure committed under profiles/ names the hash of
    the kernel sources it was captured on, and that hash is the current one:
    a figure whose kernel changed since must be recaptured or removed, never
    re-labelled."""
    import json

    import bench
    d = json.load(open(bench.TRAFFIC_FILE))
    for key, ent in d.items():
        kernel = key.split(":")[0]
        assert ent["src_sha"] == bench.gemm_source_sha(kernel), f"{key}: captured on other sources"
        assert "src_sha_note" not in ent, f"{key}: a hash must come from a capture"
