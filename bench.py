"""Benchmark of the FP8 DeepSeekMoE layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload prefill|decode|skewed]
                    [--scale-mode amax|pow2] [--gemm auto|single|pair|tall] [--balance-steps S]
                    [--impl ours|reference] [--no-cpu-baseline] [--no-e2e] [--e2e-serial]
                    [--no-extras] [--tokens T] [--experts E]

One step = the whole path over T tokens of seeded synthetic input with V3
shapes (hidden 7168, intermediate 2048, 256 routed + 1 shared experts,
top-8), weights resident in HBM: the layer forward (quantize, route, group,
gate/up GEMM + SwiGLU + requantize, down GEMM, combine) and the step's bias
update.  The update goes to a working copy of the bias, so every step routes
the batch alike; the line also reports the batch's expert load imbalance
(max / mean), the imbalance after one bias update applied for real and the
sequence-wise balance loss (alpha = 1e-4, sequences of gcd(T, 4096) tokens;
untimed), and with --balance-steps S the imbalance along S steps with the
update fed back.
With N > 1 (launched by torchrun) every rank runs its own replica of the
layer on its own batch: there is no data-path collective; timing is the max
over ranks.  Rank 0 prints one JSON line.

The end-to-end figure ("e2e") runs the same steps through host buffers:
every step copies its input in from pinned host memory and reads its output
back, on two copy streams that overlap the neighbouring steps' compute
(--e2e-serial: copies in series on the launching stream).

Unless --no-extras, the same process then measures, on the same resident
weights, the other configurations under "workloads": the decode-shaped and
the skewed layers, the standalone block-scaled GEMM at both shapes, the
device's FP8 tensor ceiling, the backward of the expert FFNs on the headline
batch and expert parallelism over 8 ranks emulated on the one GPU.

--scale-mode pow2 runs the power-of-two scale variant (scales applied by the
tensor core); the default is the pages' S = amax/448.  --gemm picks the
grouped-GEMM kernel (single CTAs by default).  --tokens / --experts shrink
the workload for profiling.  `--impl reference` times the CPU oracle (the
slow double-precision reference of the same layer) on the host cores, on a
bounded sample of the workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOADS = ("prefill", "decode", "skewed")
METRIC = "MoE-layer tokens/s and grouped FP8 GEMM TFLOP/s (% of B200 FP8 / HBM roofline)"
KERNELS_PER_STEP = 11  # quantize, router GEMM, top-k, histogram, chunk table, ranks, row copy, 2 GEMMs, combine,
#                        bias update
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
# sources each GEMM kernel is built from (the traffic figures in profiles/
# hold only while these are unchanged)
_CSRC = os.path.join(ROOT, "sparse_moe_layer_expert_b200", "csrc")
GEMM_SOURCES = {
    "gemm_fp8_kernel": [os.path.join(_CSRC, f) for f in ("gemm.cu", "gemm_tiles.cuh", "common.cuh")],
    "gemm_mx_kernel": [os.path.join(_CSRC, f) for f in ("gemm_mx.cu", "gemm_tiles.cuh", "common.cuh")],
    "gemm_pair_kernel": [os.path.join(_CSRC, f) for f in ("gemm_pair.cu", "gemm_tiles.cuh", "common.cuh")],
    "gemm_tall_kernel": [os.path.join(_CSRC, f) for f in ("gemm_tall.cu", "gemm_tiles.cuh", "common.cuh")],
}


def parse(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--workload", choices=WORKLOADS, default="prefill")
    p.add_argument("--impl", choices=("ours", "reference"), default="ours")
    p.add_argument("--seed", type=int, default=0)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-sample-tokens", type=int, default=8)
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--e2e-serial", action="store_true",
                   help="end-to-end leg with its copies in series with the compute (default: pipelined)")
    p.add_argument("--balance-steps", type=int, default=0,
                   help="after timing, run this many steps with the bias update fed back (the auxiliary-loss-free "
                        "balancing loop) and report max/mean expert load along the way")
    p.add_argument("--scale-mode", choices=("amax", "pow2"), default="amax",
                   help="amax: S = amax/448 (the pages, default); pow2: power-of-two scales applied by the "
                        "tensor core (block-scaled MMA)")
    p.add_argument("--gemm", choices=("auto", "single", "pair", "tall"), default="auto",
                   help="grouped GEMM kernel of the default scale mode: the library's choice (auto), single "
                        "CTAs, CTA pairs (tcgen05 cta_group::2) or tall tiles (256 rows x 128 weight rows)")
    p.add_argument("--no-extras", action="store_true",
                   help="skip the other workloads (decode, skewed, standalone GEMM, FP8 ceiling) measured after "
                        "the headline at N = 1")
    p.add_argument("--tokens", type=int, default=0, help="override T (profiling of smaller cases)")
    p.add_argument("--experts", type=int, default=0, help="override N_r (profiling of smaller cases)")
    return p.parse_args(argv)


# ---------------------------------------------------------------- helpers
def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Max of a per-rank scalar over all ranks (identity when world == 1)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(total_ms_max: float, steps: int, world: int, tokens_per_rank: int):
    """(ms per step, whole-job tokens/s) from the slowest rank's timed region:
    every rank processes its own batch of `tokens_per_rank` tokens per step."""
    ms_per_step = total_ms_max / steps
    return ms_per_step, world * tokens_per_rank / (ms_per_step / 1e3)


def barrier(world: int, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def workload_shape(name: str, args=None) -> dict:
    import moe_synth as S
    cfg = dict(S.CONFIGS[name])
    if args is not None and args.tokens:
        cfg["T"] = args.tokens
    if args is not None and args.experts:
        cfg["Nr"] = args.experts
        if cfg.get("n_groups"):
            cfg["n_groups"] = min(cfg["n_groups"], args.experts)
            cfg["topk_groups"] = min(cfg["topk_groups"], cfg["n_groups"])
    return cfg


def algorithmic_counts(cfg: dict, T: int, touched_routed: int) -> dict:
    """Algorithmic bytes and FLOPs of the two grouped GEMMs for one call.
    Weight bytes count every expert that receives at least one row once (the
    shared expert always); activation bytes count each (token, expert) row of
    FP8 input plus its scales once, outputs once."""
    H, I, Kr, Ns = cfg["H"], cfg["I"], cfg["Kr"], cfg.get("Ns", 1)
    rows = T * Kr + T * Ns
    E_t = touched_routed + Ns
    w13 = 2 * I * H + (2 * I // 128) * (H // 128) * 4
    w2 = H * I + (H // 128) * (I // 128) * 4
    g1_bytes = E_t * w13 + rows * (H + (H // 128) * 4) + rows * (I + (I // 128) * 4)
    g2_bytes = E_t * w2 + rows * (I + (I // 128) * 4) + rows * 4 + rows * H * 4
    g1_flops = 2.0 * rows * 2 * I * H
    g2_flops = 2.0 * rows * H * I
    return dict(g1_bytes=g1_bytes, g2_bytes=g2_bytes, g1_flops=g1_flops, g2_flops=g2_flops,
                layer_weight_bytes=E_t * (w13 + w2))


def gemm_work(M, torch, layer, T: int, stage_ms: dict, sm_mhz, kernel: int) -> dict:
    """Work of the two grouped GEMM launches of the last forward, from the
    chunk table it left in the workspace: chunks, tiles, K blocks per
    processing unit (an SM, or a pair of SMs on the CTA-pair kernel), and the
    cycles one K block took on average at the sampled SM clock.  A tile is
    128 rows x 256 weight rows (single CTA, CTA pair: 256 rows over two SMs)
    or up to 256 rows x 128 weight rows (tall tiles)."""
    pair = kernel == M.MOE_GEMM_PAIR
    tall = kernel == M.MOE_GEMM_TALL
    import math as _m
    c = layer.cfg
    ws, L = layer.workspace(T), layer.layout(T)
    nch = int(M.ws_view(ws, L, "meta", torch.int32, (4,)).cpu()[0])
    sms = torch.cuda.get_device_properties(ws.device).multi_processor_count
    units = sms // 2 if pair else sms
    out = {}
    nb1 = 2 * (c.inter // 128) if tall else c.inter // 128
    nb2 = 2 * (c.hidden // 256) if tall else (c.hidden // 128 + 1) // 2
    for name, nb, kb in (("gemm_gate_up", nb1, c.hidden // 128), ("gemm_down", nb2, c.inter // 128)):
        tiles = nch * nb
        kpu = tiles * kb / units
        d = dict(chunks=nch, tiles=tiles, k_blocks=tiles * kb, k_blocks_per_unit=round(kpu, 1),
                 unit="SM pair" if pair else "SM")
        if sm_mhz:
            d["cycles_per_k_block"] = round(stage_ms[name] * 1e-3 * sm_mhz * 1e6 / _m.ceil(kpu), 1)
        out[name] = d
    return out


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, src="fallback")


def gemm_source_sha(kernel: str) -> str:
    """Hash of the sources of a GEMM kernel ("gemm_fp8_kernel<0>" or its base name)."""
    h = hashlib.sha256()
    for f in GEMM_SOURCES[kernel.split("<")[0]]:
        h.update(open(f, "rb").read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str, kernel: str):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, or
    None when absent or taken on a different version of the GEMM source."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    d = json.load(open(TRAFFIC_FILE))
    ent = d.get(f"{kernel}:{workload}")
    if not ent or ent.get("src_sha") != gemm_source_sha(kernel):
        return None
    return float(ent["bytes_per_launch"])


class ClockSampler:
    """nvidia-smi clocks/throttle reasons sampled every 25 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu = gpu_id
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "25"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        # the region to sample starts only once the sampler is producing
        t0 = time.perf_counter()
        while self.proc is not None and time.perf_counter() - t0 < 5.0:
            if os.path.getsize(self.path) > 0 or self.proc.poll() is not None:
                break
            time.sleep(0.01)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self) -> dict:
        rows = []
        if self.path and os.path.exists(self.path):
            for line in open(self.path):
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
            os.unlink(self.path)
        if not rows:
            return dict(sm_mhz=None, sm_max_mhz=None, reasons=["unsampled"], samples=0)
        sm = sorted(float(r[1]) for r in rows if r[1].replace(".", "").isdigit())
        smax = max(float(r[2]) for r in rows if r[2].replace(".", "").isdigit())
        reasons = set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for r in rows:
            for n, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        under = [v for v in sm if v > 300] or sm
        return dict(sm_mhz=under[len(under) // 2] if under else None, sm_max_mhz=smax, reasons=sorted(reasons),
                    samples=len(rows), power_w_max=max(float(r[3]) for r in rows if _isnum(r[3])) if rows else None)


def _isnum(s):
    try:
        float(s)
        return True
    except ValueError:
        return False


# ------------------------------------------------ end to end (host buffers)
def e2e_serial(step_io, x_h, out_h, stream, dev, steps: int, world: int) -> float:
    """Steps with their copies in series on the launching stream: each step
    copies its input in from pinned host memory, runs, and reads its output
    back.  Returns the device time of `steps` steps in ms (max over ranks)."""
    import torch

    T, H = x_h.shape
    x_d = torch.empty((T, H), dtype=x_h.dtype, device=dev)
    out_d = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    barrier(world, dev)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(steps):
            x_d.copy_(x_h, non_blocking=True)
            step_io(x_d, out_d)
            out_h.copy_(out_d, non_blocking=True)
        e1.record(stream)
    torch.cuda.synchronize(dev)
    return max_over_ranks(e0.elapsed_time(e1), world, dev)


def e2e_pipelined(step_io, x_h, out_h, stream, dev, steps: int, world: int) -> float:
    """Steps with their copies overlapped, as a serving loop runs them: step
    k's input is copied in on one copy stream while step k-1 computes, and
    step k's output is read back on another while step k+1 computes.  Two
    device buffers each way; events order every reuse (step k waits for its
    input copy and for the read-back of step k-2's output from the buffer it
    writes; the input copy of step k waits until step k-2 has finished with
    its buffer).  The timed region runs on the launching stream from before
    the first input copy to after the last read-back.  out_h: two pinned
    host buffers.  Returns the device time of `steps` steps in ms (max over
    ranks)."""
    import torch

    T, H = x_h.shape
    h2d, d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    x_d = [torch.empty((T, H), dtype=x_h.dtype, device=dev) for _ in range(2)]
    out_d = [torch.empty((T, H), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    x_ready = [torch.cuda.Event() for _ in range(2)]
    computed = [torch.cuda.Event() for _ in range(2)]
    read_back = [torch.cuda.Event() for _ in range(2)]
    barrier(world, dev)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    h2d.wait_event(e0)
    d2h.wait_event(e0)
    for k in range(steps):
        b = k % 2
        with torch.cuda.stream(h2d):
            if k >= 2:
                h2d.wait_event(computed[b])
            x_d[b].copy_(x_h, non_blocking=True)
            x_ready[b].record(h2d)
        stream.wait_event(x_ready[b])
        if k >= 2:
            stream.wait_event(read_back[b])
        with torch.cuda.stream(stream):
            step_io(x_d[b], out_d[b])
        computed[b].record(stream)
        with torch.cuda.stream(d2h):
            d2h.wait_event(computed[b])
            out_h[b].copy_(out_d[b], non_blocking=True)
            read_back[b].record(d2h)
    stream.wait_stream(h2d)
    stream.wait_stream(d2h)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    return max_over_ranks(e0.elapsed_time(e1), world, dev)


# ---------------------------------------------------------- oracle (CPU)
def oracle_sample(cfg: dict, n_tok: int, seed: int, x_full, wr, bias, expert_bf16):
    """Prepare the oracle's inputs for the first n_tok tokens of the batch:
    its own quantization of the weights those tokens need (untimed set-up).
    Returns a callable that runs the timed oracle forward."""
    import numpy as np
    import oracle
    ocf = oracle.cfg(cfg["H"], cfg["I"], cfg["Nr"], cfg["Kr"], cfg.get("Ns", 1), cfg.get("n_groups", 0),
                     cfg.get("topk_groups", 0))
    x = x_full[:n_tok].cpu()
    idx, _, _, _ = oracle.route(ocf, x, wr.cpu(), bias.cpu())
    need = sorted(set(int(e) for e in idx.reshape(-1)) | set(range(cfg["Nr"], cfg["Nr"] + cfg.get("Ns", 1))))
    experts = [None] * (cfg["Nr"] + cfg.get("Ns", 1))
    for e in need:
        w13, w2 = expert_bf16(e)
        a, sa = oracle.quant_128x128(w13.cpu())
        b, sb = oracle.quant_128x128(w2.cpu())
        experts[e] = (a, sa, b, sb)
    wr_c, bias_c = wr.cpu(), bias.cpu()

    def run(threads=None):
        if threads:
            oracle.set_num_threads(threads)
        return oracle.forward(ocf, x, wr_c, bias_c, experts, tokens=np.arange(n_tok))

    return run, oracle.num_threads()


def time_oracle(run, n_tok: int, reps: int = 1, threads=None) -> float:
    if threads:
        run(threads)  # untimed: sets the thread count (and warms the caches)
    t0 = time.perf_counter()
    for _ in range(reps):
        run()
    dt = (time.perf_counter() - t0) / reps
    return n_tok / dt



# ------------------------------------------------ other workloads (same run)
def time_layer_steps(M, torch, layer, x, steps: int, warmup: int, stream, dev, gpu_id: str, bias_update=True):
    """Device time of `steps` back-to-back layer steps (forward + the step's
    bias update into a working copy of the bias) after `warmup` untimed ones,
    with per-stage times from the library's events and the SM clocks sampled
    meanwhile."""
    T = x.shape[0]
    Nr, Kr = layer.cfg.n_routed, layer.cfg.top_k
    out = torch.empty((T, layer.cfg.hidden), dtype=torch.bfloat16, device=dev)
    counts = torch.empty(Nr, dtype=torch.int32, device=dev)
    bias_next = layer.bias.clone()

    def step():
        layer.forward(x, out=out, counts_out=counts, stream=stream)
        if bias_update:
            M.moe_bias_update(bias_next, counts, Nr, T * Kr, 0.001, stream=stream)

    for _ in range(warmup):
        step()
    layer.check(stream)
    n_ev = M.MOE_PROFILE_EVENTS
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(steps)]
    ev_end = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    for row in ev:
        for e in row:
            e.record(stream)
    for e in ev_end:
        e.record(stream)
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(gpu_id)
    with sampler:
        for k in range(steps):
            M.moe_profile_events(ev[k])
            step()
            ev_end[k].record(stream)
        M.moe_profile_events(None)
        torch.cuda.synchronize(dev)
    layer.check(stream)
    stage_ms = {name: sum(ev[k][i].elapsed_time(ev[k][i + 1]) for k in range(steps)) / steps
                for i, name in enumerate(M.PROFILE_STAGES)}
    total_ms = ev[0][0].elapsed_time(ev_end[-1])
    return dict(ms_per_step=total_ms / steps, stage_ms=stage_ms, counts=counts.cpu(), clocks=sampler.summary(),
                timed_ms=total_ms)


def fp8_ceiling(torch, dev, gpu_id: str, n: int = 8192, iters: int = 20):
    """Dense FP8 (E4M3) matmul throughput of the library GEMM torch ships
    (torch._scaled_mm, per-tensor scales, bf16 out) at n^3: the device's FP8
    tensor ceiling, measured in this run.  A measurement only: nothing of the
    layer runs through it."""
    try:
        a = torch.randn((n, n), device=dev).to(torch.float8_e4m3fn)
        b = torch.randn((n, n), device=dev).to(torch.float8_e4m3fn).t()  # column-major operand
        one = torch.ones((), device=dev)
        for _ in range(3):
            torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        sampler = ClockSampler(gpu_id)
        with sampler:
            e0.record()
            for _ in range(iters):
                torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
            e1.record()
            torch.cuda.synchronize(dev)
        ms = e0.elapsed_time(e1) / iters
        del a, b
        return dict(tflops=round(2.0 * n ** 3 / (ms / 1e3) / 1e12, 1), n=n, ms=round(ms, 4),
                    how="torch._scaled_mm e4m3 x e4m3 -> bf16, per-tensor scales, %d back-to-back" % iters,
                    clocks=sampler.summary())
    except Exception as exc:  # report why instead of failing the bench
        return dict(tflops=None, error=str(exc).splitlines()[0][:160])


def time_blockscaled_gemm(M, torch, S, dev, gpu_id: str, Mrows: int, K: int, N: int, seed: int, steps: int,
                          warmup: int, copies: int = 8):
    """The standalone fine-grained block-scaled GEMM (fp8_blockscaled_gemm) at
    [M, K] x [K, N]: A ~ N(0,1) with 1% outliers x50 quantized 1x128, B ~
    N(0, 0.02^2) quantized 128x128 (passed as [N, K]); `copies` quantized
    copies of B are used in turn so that B streams from HBM every call."""
    a = S.gen_gemm_a(Mrows, K, seed, device=dev)
    A, sA = M.fp8_quant_1x128(a)
    bs = []
    for c in range(copies):
        bt = S.gen_gemm_b(K, N, seed + 101 * c, device=dev).t().contiguous()
        bs.append(M.fp8_quant_128x128(bt))
        del bt
    C = torch.empty((Mrows, N), dtype=torch.bfloat16, device=dev)
    err = M.new_err_flag(dev)
    for i in range(warmup):
        M.fp8_blockscaled_gemm(A, sA, bs[i % copies][0], bs[i % copies][1], C=C, err=err)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(gpu_id)
    with sampler:
        e0.record()
        for i in range(steps):
            M.fp8_blockscaled_gemm(A, sA, bs[i % copies][0], bs[i % copies][1], C=C, err=err)
        e1.record()
        torch.cuda.synchronize(dev)
    st, v = M.moe_check_device_error(err)
    if st != M.MOE_OK:
        raise M.MoeError(st, f"fp8_blockscaled_gemm device error {v:#x}")
    ms = e0.elapsed_time(e1) / steps
    flops = 2.0 * Mrows * N * K
    return dict(ms=round(ms, 4), tflops=round(flops / (ms / 1e3) / 1e12, 1), flops=flops, clocks=sampler.summary(),
                l2="B rotated over %d quantized copies (%.0f MB)" % (copies, copies * N * K / 1e6))


def time_backward(M, torch, S, layer, x, seed: int, stream, dev, gpu_id: str, peaks: dict, fp8_peak: float,
                  fp8_src: str, steps: int = 5, warmup: int = 2) -> dict:
    """Device time of moe_backward (routing held fixed) for the batch x that
    the layer's last forward routed: G, U recomputed, the dgrad GEMMs
    against the transposed weights (made once, set-up), the SwiGLU backward,
    dx and every expert's FP32 weight gradients.  Algorithmic work: five
    GEMMs of 2 * RS * H * I multiply-adds each counted in units of the down
    projection (recompute 2, dh 1, dx 2, dW2 1, dW13 2: 16 RS H I flops);
    bytes: the FP32 weight gradients written ([E, 3 I, H]) plus the weights
    read twice (forward copy and transposed copy)."""
    c = layer.cfg
    H, I, E = c.hidden, c.inter, c.n_routed + c.n_shared
    T = x.shape[0]
    RS = T * c.top_k + T * c.n_shared
    dout = S.gen_x(T, H, seed * 1009 + 23, device=dev)
    dx = torch.empty((T, H), dtype=torch.float32, device=dev)
    dW13 = torch.empty((E, 2 * I, H), dtype=torch.float32, device=dev)
    dW2 = torch.empty((E, H, I), dtype=torch.float32, device=dev)
    layer.forward(x, stream=stream)
    wt = M.moe_transpose_weights(c, layer.weights(), stream=stream)
    bws = layer.backward_workspace(T)

    def bwd():
        M.moe_backward(c, layer.weights(), wt, x, dout, layer.workspace(T), dx=dx, dW13=dW13, dW2=dW2, ws=bws,
                       err=layer.err, stream=stream)

    for _ in range(warmup):
        bwd()
    layer.check(stream)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    nf, nb = M.MOE_PROFILE_EVENTS, M.MOE_PROFILE_BWD_EVENTS
    sev = [[torch.cuda.Event(enable_timing=True) for _ in range(nf + nb)] for _ in range(steps)]
    for e in ev + [e for row in sev for e in row]:
        e.record(stream)
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(gpu_id)
    with sampler:
        ev[0].record(stream)
        for k in range(steps):
            M.moe_profile_events(sev[k])
            bwd()
            ev[k + 1].record(stream)
        M.moe_profile_events(None)
        torch.cuda.synchronize(dev)
    layer.check(stream)
    ms = ev[0].elapsed_time(ev[-1]) / steps
    stage_ms = {name: round(sum(sev[k][nf + i].elapsed_time(sev[k][nf + i + 1]) for k in range(steps)) / steps, 4)
                for i, name in enumerate(M.PROFILE_BWD_STAGES)}
    flops = 16.0 * RS * H * I
    wbytes = E * 3 * I * H * 4 + 2 * E * 3 * I * H
    tfl = flops / (ms / 1e3) / 1e12
    gbs = wbytes / (ms / 1e3) / 1e9
    t_tc, t_mem = flops / (fp8_peak * 1e12), wbytes / (peaks["hbm"] * 1e9)
    out = dict(workload=f"backward of the expert FFNs: T={T} H={H} I={I} E={E} (routing of the prefill batch held "
                        "fixed), FP32 dx and weight gradients",
               ms=round(ms, 4), tflops=round(tfl, 1), frac_fp8=round(tfl / fp8_peak, 4), fp8_peak=fp8_peak,
               fp8_peak_src=fp8_src, algorithmic_flops=flops, weight_gradient_and_weight_bytes=wbytes,
               achieved_gbs=round(gbs, 1), frac_hbm=round(gbs / peaks["hbm"], 4),
               bound="hbm" if t_mem >= t_tc else "tensor",
               roofline_ms=round(max(t_tc, t_mem) * 1e3, 4), stage_ms=stage_ms, clocks=sampler.summary())
    del dW13, dW2, dx, wt
    torch.cuda.empty_cache()
    return out


def time_ep_emulated(M, torch, S, layer, seed: int, stream, dev, W: int = 8, T: int = 4096, reps: int = 3) -> dict:
    """The expert-parallel forward of W ranks (T tokens each; rank d owns
    routed experts [d N_r/W, (d+1) N_r/W)) with all W ranks' work run on this
    one GPU (sparse_moe_layer_expert_b200.ep.LibraryOps; the all-to-all
    exchanges are device copies between the ranks' buffers).  Device time of
    each phase from CUDA events around it, summed over the ranks and divided
    by W: the compute one rank of a W-GPU run does per layer.  The bytes each
    rank would send and receive over NVLink give the exchange time at the
    pool's measured 770 GB/s per direction (a projection: no NVLink here)."""
    from sparse_moe_layer_expert_b200.ep import LibraryOps, LocalExchange
    ops = [LibraryOps(layer, W, r) for r in range(W)]
    xs = [S.gen_x(T, layer.cfg.hidden, seed * 1009 + 31 + r, device=dev) for r in range(W)]
    H = layer.cfg.hidden
    phases = ("quant_route", "dispatch", "exchange_rows", "experts", "exchange_back", "shared", "combine")
    acc = {k: 0.0 for k in phases}

    def timed(name, fn):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        r = fn()
        e1.record(stream)
        return r, (name, e0, e1)

    sent = back_bytes = 0
    for it in range(reps + 1):  # the first round is a warm-up
        evs = []
        st, disp = [], []
        for r in range(W):
            v, e = timed("quant_route", lambda: ops[r].quant_route(xs[r]))
            st.append(v)
            evs.append(e)
        for r in range(W):
            v, e = timed("dispatch", lambda: ops[r].dispatch(*st[r]))
            disp.append(v)
            evs.append(e)
        send_counts = [d[1] for d in disp]
        recv, e = timed("exchange_rows", lambda: LocalExchange.rows([d[0] for d in disp], send_counts))
        evs.append(e)
        partial = []
        for d in range(W):
            v, e = timed("experts", lambda: ops[d].experts(recv[d]))
            partial.append(v)
            evs.append(e)
        recv_counts = LocalExchange.counts(send_counts)
        back, e = timed("exchange_back", lambda: LocalExchange.rows(partial, recv_counts))
        evs.append(e)
        for r in range(W):
            y_sh, e = timed("shared", lambda: ops[r].shared(disp[r][3]))
            evs.append(e)
            _, e = timed("combine", lambda: ops[r].combine(xs[r], disp[r][2], back[r], y_sh))
            evs.append(e)
        torch.cuda.synchronize(dev)
        layer.check(stream)
        if it > 0:
            for name, e0, e1 in evs:
                acc[name] += e0.elapsed_time(e1) / reps
        sent = sum(sum(c) - c[r] for r, c in enumerate(send_counts)) / W
        back_bytes = sent * H * 2
    row_bytes = M.moe_ep_row_bytes(layer.cfg)
    per_rank = {k: round(v / W, 4) for k, v in acc.items()}
    compute = sum(v for k, v in per_rank.items() if not k.startswith("exchange"))
    nvl = 770.0
    t_send = sent * row_bytes / (nvl * 1e9) * 1e3
    t_back = back_bytes / (nvl * 1e9) * 1e3
    return dict(workload=f"expert parallelism emulated on one GPU: W={W} ranks x T={T} tokens, V3 layer, rank d owns "
                         f"{layer.cfg.n_routed // W} routed experts",
                ms_per_rank=per_rank, compute_ms_per_rank=round(compute, 4),
                tokens_per_s_per_rank_compute=round(T / (compute / 1e3), 1),
                rows_sent_to_other_ranks_per_rank=round(sent, 1), row_bytes=row_bytes,
                nvlink_projection_ms=dict(send=round(t_send, 4), back=round(t_back, 4),
                                          how="bytes one rank sends to the other ranks / 770 GB/s per direction "
                                              "(the pool's measured peer copy); the exchanges here are device "
                                              "copies, not NVLink"))


def extra_workloads(M, torch, S, layer, args, seed: int, stream, dev, gpu_id: str, peaks: dict, x=None) -> dict:
    """The other configurations of the workload set, measured in the same
    process on the same resident expert weights: the decode-shaped layer
    (T = 64, zero bias), the skewed layer (T = 16384, mixture input,
    group-limited routing 8 x 32 / top-4 groups, zero bias, then one bias
    update), the standalone block-scaled GEMM at both shapes and the device's
    FP8 tensor ceiling; then the backward of the expert FFNs on the headline
    batch x (FP32 gradients; default scale mode only)."""
    H, I, Nr, Kr = layer.cfg.hidden, layer.cfg.inter, layer.cfg.n_routed, layer.cfg.top_k
    res = {}
    ceil = fp8_ceiling(torch, dev, gpu_id)
    res["fp8_ceiling"] = ceil
    fp8_peak = ceil.get("tflops") or 2.0 * peaks["bf16"]
    fp8_src = "measured in this run (torch._scaled_mm)" if ceil.get("tflops") else \
        peaks["src"] + " bf16 burst x 2 (nominal FP8/bf16 ratio)"
    # decode: T = 64, zero bias
    dec = S.CONFIGS["decode"]
    zero = torch.zeros(Nr, dtype=torch.float32, device=dev)
    lay_d = layer.sibling(bias=zero)
    x_d = S.gen_x(dec["T"], H, seed * 1009 + 7, device=dev)
    r = time_layer_steps(M, torch, lay_d, x_d, args.steps, args.warmup, stream, dev, gpu_id)
    touched = int((r["counts"] > 0).sum())
    alg = algorithmic_counts(dict(dec), dec["T"], touched)
    layer_bytes = alg["layer_weight_bytes"] + Nr * H * 2 + dec["T"] * H * 2 * 2
    res["decode"] = dict(
        workload=f"decode: T={dec['T']} H={H} I={I} Nr={Nr} Kr={Kr} Ns=1, zero bias",
        ms_per_step=round(r["ms_per_step"], 4), tokens_per_s=round(dec["T"] / (r["ms_per_step"] / 1e3), 1),
        experts_touched=touched + 1,
        layer_hbm=dict(algorithmic_bytes=layer_bytes, achieved_gbs=round(layer_bytes / (r["ms_per_step"] / 1e3) / 1e9, 1),
                       frac=round(layer_bytes / (r["ms_per_step"] / 1e3) / 1e9 / peaks["hbm"], 4),
                       peak=peaks["hbm"], how="expert weights touched + router weights + x in/out over the whole "
                                            "step (layer + bias update) / HBM copy peak"),
        gate_up_hbm_frac=round(alg["g1_bytes"] / (r["stage_ms"]["gemm_gate_up"] / 1e3) / 1e9 / peaks["hbm"], 4),
        stage_ms={k: round(v, 4) for k, v in r["stage_ms"].items()}, clocks=r["clocks"])
    del lay_d, x_d
    # skewed: T = 16384, mixture input, group-limited routing, zero bias
    sk = S.CONFIGS["skewed"]
    lay_s = layer.sibling(bias=zero.clone(), n_groups=sk["n_groups"], topk_groups=sk["topk_groups"])
    x_s, _ = S.gen_mixture_x(sk["T"], H, seed * 1009 + 11, device=dev)
    r = time_layer_steps(M, torch, lay_s, x_s, args.steps, args.warmup, stream, dev, gpu_id)
    Ts = sk["T"]
    mean = Ts * Kr / Nr
    c0 = r["counts"]
    lay_s.bias_update(c0.to(dev), Ts)  # one update b_i -/+ 0.001 applied for real
    c1 = torch.empty(Nr, dtype=torch.int32, device=dev)
    lay_s.forward(x_s, counts_out=c1, stream=stream)
    lay_s.check(stream)
    touched = int((c0 > 0).sum())
    alg = algorithmic_counts(dict(sk), Ts, touched)
    g_ms = r["stage_ms"]["gemm_gate_up"] + r["stage_ms"]["gemm_down"]
    tfl = (alg["g1_flops"] + alg["g2_flops"]) / (g_ms / 1e3) / 1e12
    res["skewed"] = dict(
        workload=f"skewed: T={Ts} H={H} I={I} Nr={Nr} Kr={Kr} Ns=1, groups {sk['n_groups']}/{sk['topk_groups']}, "
                 "32-centroid Zipf(1) mixture input, zero bias",
        ms_per_step=round(r["ms_per_step"], 4), tokens_per_s=round(Ts / (r["ms_per_step"] / 1e3), 1),
        load_max_over_mean=round(float(c0.max()) / mean, 3),
        after_one_bias_update=round(float(c1.max().item()) / mean, 3),
        grouped_gemm_tflops=round(tfl, 1), grouped_gemm_frac_fp8=round(tfl / fp8_peak, 4), fp8_peak=fp8_peak,
        fp8_peak_src=fp8_src, frac_of_nominal_4500=round(tfl / 4500.0, 4),
        stage_ms={k: round(v, 4) for k, v in r["stage_ms"].items()}, clocks=r["clocks"])
    del lay_s, x_s
    torch.cuda.empty_cache()
    # the standalone block-scaled GEMM at both shapes
    for (Mr, K, N) in S.GEMM_SHAPES:
        g = time_blockscaled_gemm(M, torch, S, dev, gpu_id, Mr, K, N, seed, args.steps, args.warmup)
        g.update(frac_fp8=round(g["tflops"] / fp8_peak, 4), fp8_peak=fp8_peak, fp8_peak_src=fp8_src,
                 frac_of_nominal_4500=round(g["tflops"] / 4500.0, 4))
        res[f"gemm_M{Mr}_K{K}_N{N}"] = g
        torch.cuda.empty_cache()
    if x is not None and layer.cfg.scale_mode == M.MOE_SCALE_AMAX:
        res["backward"] = time_backward(M, torch, S, layer, x, seed, stream, dev, gpu_id, peaks, fp8_peak, fp8_src)
    if layer.cfg.n_routed % 8 == 0 and layer.cfg.n_shared == 1:
        res["expert_parallel_emulated"] = time_ep_emulated(M, torch, S, layer, seed, stream, dev)
        torch.cuda.empty_cache()
    return res


# ------------------------------------------------------------------ main
def main(argv=None):
    args = parse(argv)
    rank, world, local = dist_env()
    if args.impl == "reference":
        return run_reference(args, rank, world)
    import torch
    import torch.distributed as dist

    import moe_synth as S
    import sparse_moe_layer_expert_b200 as M

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    M.moe_set_gemm_variant({"auto": M.MOE_GEMM_AUTO, "single": M.MOE_GEMM_SINGLE, "pair": M.MOE_GEMM_PAIR,
                            "tall": M.MOE_GEMM_TALL}[args.gemm])
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    cfg = workload_shape(args.workload, args)
    T = cfg["T"]
    shape = {k: cfg[k] for k in ("H", "I", "Nr", "Kr", "Ns", "n_groups", "topk_groups")}
    shape["scale_mode"] = M.MOE_SCALE_POW2 if args.scale_mode == "pow2" else M.MOE_SCALE_AMAX
    seed = args.seed

    def expert_bf16(e):
        return S.gen_expert(e, cfg["H"], cfg["I"], seed, device=dev)

    wr = S.gen_router(cfg["Nr"], cfg["H"], seed, device=dev)
    bias = S.gen_bias(cfg["Nr"], seed, cfg.get("bias", "uniform"), device=dev)
    layer = M.MoeLayer.from_generator(shape, expert_bf16, wr, bias, device=dev)
    xseed = seed * 1009 + rank
    if cfg.get("x") == "mixture":
        x, _ = S.gen_mixture_x(T, cfg["H"], xseed, device=dev)
    else:
        x = S.gen_x(T, cfg["H"], xseed, device=dev)
    out = torch.empty((T, cfg["H"]), dtype=torch.bfloat16, device=dev)
    counts = torch.empty(cfg["Nr"], dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    # A step is the whole path: the layer forward, then the bias update of
    # the step (b_i -/+ gamma by the step's expert loads).  The update is
    # written to a working copy of the bias, so every timed step routes the
    # batch with the same bias (stationary routing) while doing all of the
    # update's work.
    bias_next = layer.bias.clone()
    total_assign = T * cfg["Kr"]

    def step(x_in):
        layer.forward(x_in, out=out, counts_out=counts, stream=stream)
        M.moe_bias_update(bias_next, counts, cfg["Nr"], total_assign, 0.001, stream=stream)

    def step_io(x_in, out_buf):  # the same step, output to a given buffer (end-to-end legs)
        layer.forward(x_in, out=out_buf, counts_out=counts, stream=stream)
        M.moe_bias_update(bias_next, counts, cfg["Nr"], total_assign, 0.001, stream=stream)

    torch.cuda.synchronize(dev)

    # ------------------------------------------------ device-timed steps
    for _ in range(args.warmup):
        step(x)
    layer.check(stream)
    n_ev = M.MOE_PROFILE_EVENTS
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(args.steps)]
    ev_end = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]  # after each step's bias update
    for row in ev:  # torch creates the CUDA event on first record; the library needs the handles
        for e in row:
            e.record(stream)
    for e in ev_end:
        e.record(stream)
    barrier(world, dev)
    torch.cuda.synchronize(dev)
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:  # older torch: fall back to the ordinal
        gpu_id = str(local)
    sampler = ClockSampler(gpu_id)
    with sampler:
        for k in range(args.steps):
            M.moe_profile_events(ev[k])
            step(x)
            ev_end[k].record(stream)
        M.moe_profile_events(None)
        torch.cuda.synchronize(dev)
    barrier(world, dev)
    layer.check(stream)
    clocks = sampler.summary()
    step_ms = [ev[k][0].elapsed_time(ev_end[k]) for k in range(args.steps)]
    stage_ms = {name: sum(ev[k][i].elapsed_time(ev[k][i + 1]) for k in range(args.steps)) / args.steps
                for i, name in enumerate(M.PROFILE_STAGES)}
    stage_ms["bias_update"] = sum(ev[k][n_ev - 1].elapsed_time(ev_end[k]) for k in range(args.steps)) / args.steps
    # the timed region is the K back-to-back steps: first start to last end
    total_ms = ev[0][0].elapsed_time(ev_end[-1])
    total_ms = max_over_ranks(total_ms, world, dev)
    ms_per_step, value = aggregate(total_ms, args.steps, world, T)

    counts_h = counts.cpu()
    touched = int((counts_h > 0).sum())
    gemm_kernel = M.moe_gemm_kernel_for(layer.cfg, T)
    work = gemm_work(M, torch, layer, T, stage_ms, clocks.get("sm_mhz"), gemm_kernel)
    # sequence-wise balance loss (alpha = 1e-4) of the batch the timed steps
    # routed, read from the last forward's workspace before anything reroutes
    seq_len = math.gcd(T, 4096)
    seq_loss = layer.seq_balance_loss(T, seq_len, 1e-4, stream=stream).cpu().tolist()
    # expert load imbalance of the batch, and after one bias update applied
    # for real (the same batch routed again with b - gamma * sign(load - mean))
    mean_load = total_assign / cfg["Nr"]
    b_upd = layer.bias.clone()
    M.moe_bias_update(b_upd, counts, cfg["Nr"], total_assign, 0.001, stream=stream)
    b_keep, layer.bias = layer.bias, b_upd
    counts_upd = torch.empty_like(counts)
    layer.forward(x, out=out, counts_out=counts_upd, stream=stream)
    layer.bias = b_keep
    load = dict(max_over_mean=round(float(counts_h.max()) / mean_load, 3),
                after_one_bias_update=round(float(counts_upd.max().item()) / mean_load, 3),
                seq_balance_loss=dict(alpha=1e-4, seq_len=seq_len,
                                      values=[float(f"{v:.6g}") for v in seq_loss[:8]]))
    alg = algorithmic_counts(cfg, T, touched)
    peaks = measured_peaks()
    g1_ms, g2_ms = stage_ms["gemm_gate_up"], stage_ms["gemm_down"]
    dom = "gemm_gate_up" if g1_ms >= g2_ms else "gemm_down"
    dom_ms = max(g1_ms, g2_ms)
    dom_bytes = alg["g1_bytes"] if dom == "gemm_gate_up" else alg["g2_bytes"]
    dom_flops = alg["g1_flops"] if dom == "gemm_gate_up" else alg["g2_flops"]
    # FP8 dense = 2 x bf16 (nominal ratio 4.5 / 2.25 PFLOP/s); the burst figure
    # for a timed region under a second, the sustained one for longer ones
    sustained = total_ms > 1000.0
    fp8_peak = 2.0 * (peaks["bf16_sustained"] if sustained else peaks["bf16"])
    fp8_src = peaks["src"] + (" bf16 sustained x 2" if sustained else " bf16 burst x 2")
    t_mem = dom_bytes / (peaks["hbm"] * 1e9)
    t_tc = dom_flops / (fp8_peak * 1e12)
    kname = {M.MOE_GEMM_BLOCK_SCALED: "gemm_mx_kernel", M.MOE_GEMM_PAIR: "gemm_pair_kernel",
             M.MOE_GEMM_TALL: "gemm_tall_kernel"}.get(gemm_kernel, "gemm_fp8_kernel")
    kernel_name = f"{kname}<0>" if dom == "gemm_gate_up" else f"{kname}<1>"
    if t_mem >= t_tc:
        achieved = dom_bytes / (dom_ms / 1e3) / 1e9
        roofline = dict(bound="hbm", achieved=round(achieved, 1), peak=peaks["hbm"], unit="GB/s",
                        frac=round(achieved / peaks["hbm"], 4), traffic=profiled_traffic(args.workload, kernel_name),
                        kernel=dom, peak_src=peaks["src"] + " (HBM copy)", algorithmic_bytes=dom_bytes)
    else:
        achieved = dom_flops / (dom_ms / 1e3) / 1e12
        roofline = dict(bound="tensor", achieved=round(achieved, 1), peak=round(fp8_peak, 1), unit="TFLOP/s",
                        frac=round(achieved / fp8_peak, 4), traffic=profiled_traffic(args.workload, kernel_name),
                        kernel=dom, peak_src=fp8_src,
                        algorithmic_flops=dom_flops)
    gemm_tflops = (alg["g1_flops"] + alg["g2_flops"]) / ((g1_ms + g2_ms) / 1e3) / 1e12

    # ------------------------------------------------ end to end (host buffers)
    e2e = None
    if not args.no_e2e:
        x_h = x.cpu().pin_memory()
        out_h = [torch.empty((T, cfg["H"]), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        mode, note = ("serial", "requested") if args.e2e_serial else ("pipelined", None)
        e2e_ms = None
        if mode == "pipelined":
            try:
                for _ in range(max(1, args.warmup // 2)):
                    e2e_pipelined(step_io, x_h, out_h, stream, dev, 2, world)
                e2e_ms = e2e_pipelined(step_io, x_h, out_h, stream, dev, args.steps, world) / args.steps
                # every step still holds its whole computation: a shorter
                # step than the device-only one means the loop is broken
                if e2e_ms < 0.98 * ms_per_step:
                    mode, note, e2e_ms = "serial", f"pipelined loop measured {e2e_ms:.3f} ms/step < device", None
            except Exception as exc:  # measure serially instead; the line says why
                torch.cuda.synchronize(dev)
                mode, note, e2e_ms = "serial", f"pipelined loop failed: {str(exc).splitlines()[0][:120]}", None
        if e2e_ms is None:
            for _ in range(max(1, args.warmup // 2)):
                e2e_serial(step_io, x_h, out_h[0], stream, dev, 1, world)
            e2e_ms = e2e_serial(step_io, x_h, out_h[0], stream, dev, args.steps, world) / args.steps
        e2e = dict(value=round(world * T / (e2e_ms / 1e3), 1), unit="tokens/s",
                   h2d_bytes_per_step=x_h.numel() * x_h.element_size(),
                   d2h_bytes_per_step=out_h[0].numel() * out_h[0].element_size(), ms_per_step=round(e2e_ms, 4),
                   copies=mode)
        if note:
            e2e["note"] = note
        layer.check(stream)

    # ------------------------------------------------ balancing loop (untimed)
    balance = None
    if args.balance_steps > 0:
        b_keep = layer.bias.clone()
        marks = sorted({0, 1, 2, 5, 10, 20, 50, 100, 200, 500, 1000, args.balance_steps} & set(range(args.balance_steps + 1)))
        traj = {}
        for k in range(args.balance_steps + 1):
            layer.forward(x, out=out, counts_out=counts, stream=stream)
            if k in marks:
                traj[k] = round(float(counts.max().item()) / mean_load, 3)
            if k < args.balance_steps:
                M.moe_bias_update(layer.bias, counts, cfg["Nr"], total_assign, 0.001, stream=stream)
        layer.bias.copy_(b_keep)
        layer.check(stream)
        balance = dict(gamma=0.001, steps=args.balance_steps, max_over_mean={str(k): v for k, v in traj.items()})

    # ------------------------------------------------ other workloads (N = 1)
    extras = None
    if world == 1 and not args.no_extras and args.workload == "prefill" and not args.tokens and not args.experts:
        extras = extra_workloads(M, torch, S, layer, args, seed, stream, dev, gpu_id, peaks, x=x)

    # ------------------------------------------------ CPU oracle baseline
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        n = args.cpu_sample_tokens
        run, threads = oracle_sample(cfg, n, seed, x, wr, bias, expert_bf16)
        used = int(min(threads, n))  # the oracle parallelises over tokens
        tps = time_oracle(run, n)
        tps1 = time_oracle(run, n, threads=1)
        run(threads)
        cpu = dict(value=round(tps, 4), unit="tokens/s", cores=used, kind="oracle", nproc=os.cpu_count(),
                   threads_used=used, one_thread_value=round(tps1, 4),
                   sample=f"first {n} tokens of the {args.workload} batch: full layer (quantize, route over all "
                          f"{cfg['Nr']} experts, shared + top-{cfg['Kr']} FP8 FFNs, combine), OpenMP over the "
                          f"tokens ({used} threads; one_thread_value with 1); weight quantization by the oracle "
                          f"excluded (set-up)")

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0
    line = dict(
        metric=METRIC, value=round(value, 1), unit="tokens/s", n_gpus=world, steps=args.steps, warmup=args.warmup,
        ms_per_step=round(ms_per_step, 4), higher_is_better=True, scaling="weak", vs_baseline=None, dtype="e4m3",
        data="synthetic",
        config=dict(workload=f"{args.workload}: T={T} H={cfg['H']} I={cfg['I']} Nr={cfg['Nr']} Kr={cfg['Kr']} "
                             f"Ns={cfg.get('Ns', 1)} groups={cfg.get('n_groups', 0)}/{cfg.get('topk_groups', 0)}",
                    global_batch=world * T, tokens_per_gpu=T, parallelism=f"replicas x{world} (no collective)",
                    l2="no flush: per-step working set >= 11 GB of expert weights >> 126 MB L2",
                    scales="amax/448 (FP32 promotion per 128-K block)" if args.scale_mode == "amax" else
                    "power of two (applied by the tensor core, block-scaled MMA)",
                    gemm_kernel=kname,
                    seed=seed),
        roofline=roofline,
        grouped_gemm_tflops=round(gemm_tflops, 1),
        grouped_gemm_frac_fp8_peak=round(gemm_tflops / fp8_peak, 4),
        fp8_peak=dict(tflops=fp8_peak, src=fp8_src),
        layer_weight_gb=round(alg["layer_weight_bytes"] / 1e9, 3),
        experts_touched=touched + cfg.get("Ns", 1),
        load=load,
        **({"balance": balance} if balance else {}),
        stage_ms={k: round(v, 4) for k, v in stage_ms.items()},
        gemm_work=work,
        step_ms_min=round(min(step_ms), 4),
        cpu_baseline=cpu,
        e2e=e2e,
        **({"workloads": extras} if extras else {}),
        gpu_launches=KERNELS_PER_STEP * args.steps,
        clocks=clocks,
    )
    print(json.dumps(line), flush=True)
    return 0


def run_reference(args, rank: int, world: int) -> int:
    """The reference arm: the CPU oracle, timed on the host cores, on a
    bounded sample (a few tokens per step) of the same workload."""
    if rank != 0:
        return 0
    import torch

    import moe_synth as S
    cfg = workload_shape(args.workload, args)
    T = cfg["T"]
    seed = args.seed
    dev = "cuda" if torch.cuda.is_available() else "cpu"

    def expert_bf16(e):
        return S.gen_expert(e, cfg["H"], cfg["I"], seed, device=dev)

    wr = S.gen_router(cfg["Nr"], cfg["H"], seed, device=dev)
    bias = S.gen_bias(cfg["Nr"], seed, cfg.get("bias", "uniform"), device=dev)
    if cfg.get("x") == "mixture":
        x, _ = S.gen_mixture_x(T, cfg["H"], seed * 1009, device=dev)
    else:
        x = S.gen_x(T, cfg["H"], seed * 1009, device=dev)
    n = max(1, min(args.cpu_sample_tokens, 4))
    run, threads = oracle_sample(cfg, n, seed, x, wr, bias, expert_bf16)
    for _ in range(args.warmup):
        run()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run()
    dt = (time.perf_counter() - t0) / args.steps
    tps = n / dt
    sample = (f"{n} tokens of the {args.workload} batch per step (full layer: quantize, route, shared + "
              f"top-{cfg['Kr']} FFNs, combine); oracle weight quantization excluded")
    line = dict(impl="reference", metric=METRIC, value=round(tps, 4), unit="tokens/s", n_gpus=world,
                steps=args.steps, warmup=args.warmup, ms_per_step=round(dt * 1e3, 2), higher_is_better=True,
                scaling="weak", vs_baseline=None, dtype="f64", data="synthetic",
                config=dict(workload=f"{args.workload}: T={T} H={cfg['H']} I={cfg['I']} Nr={cfg['Nr']} "
                                     f"Kr={cfg['Kr']} Ns={cfg.get('Ns', 1)}", global_batch=n),
                cpu_baseline=dict(kind="oracle", cores=int(min(threads, n)), sample=sample, value=round(tps, 4),
                                  unit="tokens/s"),
                e2e=dict(value=round(tps, 4), unit="tokens/s", h2d_bytes_per_step=0, d2h_bytes_per_step=0))
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
