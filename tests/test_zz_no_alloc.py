"""moe_route_noalloc: the router for callers that cannot allocate device
memory (a host that owns all device memory through its own planner, or a
latency-critical path that cannot afford an allocation's implicit device
synchronisation).  It keeps its scratch in a fixed array inside the library.

Called through the C ABI (ctypes) and compared with moe_route, which takes
a caller-provided workspace, on two calls in a row: expert indices and counts
must be identical, gates within the router's tolerance.  Works alone in a
fresh process and after the other tests (the scratch keeps the previous
call's contents, which the router overwrites before reading)."""
import ctypes as C

import numpy as np
import pytest
import torch

import moe_synth as S

pytestmark = pytest.mark.gpu


def _inputs(cfg, T, seed):
    x = S.gen_x(T, cfg["H"], seed, device="cuda")
    wr = S.gen_router(cfg["Nr"], cfg["H"], seed, device="cuda")
    bias = S.gen_bias(cfg["Nr"], seed, cfg.get("bias", "uniform"), device="cuda")
    return x, wr, bias


@pytest.mark.parametrize("name,T", [("tiny", 256), ("tiny", 129), ("decode", 64), ("prefill", 4096)])
def test_noalloc_matches_workspace_router_twice(name, T):
    import sparse_moe_layer_expert_b200 as m
    cfg = dict(S.CONFIGS[name])
    mc = m.config_from(cfg)
    x, wr, bias = _inputs(cfg, T, 40 + T)
    err = m.new_err_flag()
    ref_idx, ref_gate, ref_counts = m.moe_route(mc, x, wr, bias, err=err)
    torch.cuda.synchronize()
    for call in range(2):
        idx = torch.full((T, cfg["Kr"]), -1, dtype=torch.int32, device="cuda")
        gate = torch.full((T, cfg["Kr"]), -1.0, dtype=torch.float32, device="cuda")
        counts = torch.full((cfg["Nr"],), -7, dtype=torch.int32, device="cuda")
        st = m.lib.moe_route_noalloc(C.byref(mc), x.data_ptr(), wr.data_ptr(), bias.data_ptr(), T, idx.data_ptr(),
                                     gate.data_ptr(), counts.data_ptr(), err.data_ptr(),
                                     torch.cuda.current_stream().cuda_stream)
        assert st == m.MOE_OK, m.lib.moe_status_string(st)
        assert m.moe_check_device_error(err) == (m.MOE_OK, 0)
        assert torch.equal(idx, ref_idx), f"call {call}: expert indices differ"
        assert torch.equal(counts, ref_counts), f"call {call}: counts differ"
        assert np.allclose(gate.cpu().numpy(), ref_gate.cpu().numpy(), rtol=0, atol=2e-6), f"call {call}: gates"


def test_noalloc_rejects_calls_beyond_its_scratch():
    import sparse_moe_layer_expert_b200 as m
    cfg = dict(S.PREFILL)
    mc = m.config_from(cfg)
    T = 20000  # 20000 x 256 FP32 partial logits exceed the 16 MiB scratch
    assert m.moe_route_workspace_size(mc, T) - 256 > m.MOE_ROUTE_NOALLOC_SCRATCH_BYTES
    assert m.moe_route_workspace_size(mc, 8192) - 256 <= m.MOE_ROUTE_NOALLOC_SCRATCH_BYTES
    x = torch.zeros((T, cfg["H"]), dtype=torch.bfloat16, device="cuda")
    wr = torch.zeros((cfg["Nr"], cfg["H"]), dtype=torch.bfloat16, device="cuda")
    bias = torch.zeros(cfg["Nr"], device="cuda")
    idx = torch.empty((T, cfg["Kr"]), dtype=torch.int32, device="cuda")
    gate = torch.empty((T, cfg["Kr"]), device="cuda")
    counts = torch.empty(cfg["Nr"], dtype=torch.int32, device="cuda")
    err = m.new_err_flag()
    st = m.lib.moe_route_noalloc(C.byref(mc), x.data_ptr(), wr.data_ptr(), bias.data_ptr(), T, idx.data_ptr(),
                                 gate.data_ptr(), counts.data_ptr(), err.data_ptr(),
                                 torch.cuda.current_stream().cuda_stream)
    assert st == m.MOE_ERR_WORKSPACE_TOO_SMALL
