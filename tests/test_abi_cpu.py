"""The C-ABI library loads without a GPU, exports every entry point that
include/moe_fp8.h declares, and validates arguments on the host (no compute
call is made here)."""
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_fp8.h")


@pytest.fixture(scope="module")
def m():
    import sparse_moe_layer_expert_b200 as pkg
    return pkg


def declared_functions():
    txt = open(HEADER).read()
    return re.findall(r"^MOE_API\s+[a-z_ 0-9]+?\**\s*([a-z_0-9]+)\(", txt, flags=re.M)


def test_every_declared_symbol_is_exported(m):
    names = declared_functions()
    assert len(names) >= 14
    for n in names:
        assert hasattr(m.lib, n), n
    assert set(names) == set(m.EXPORTS)


def test_status_strings_and_version(m):
    assert m.lib.moe_abi_version() == 104
    assert m.lib.moe_status_string(0) == b"ok"
    assert b"128" in m.lib.moe_status_string(m.MOE_ERR_UNSUPPORTED_SHAPE)
    assert m.lib.moe_status_string(12345) == b"unknown status"


def test_host_validation_without_device(m):
    L = m.lib
    # shape errors are reported before any device query
    assert L.fp8_quant_1x128(None, 4, 100, 128, None, None, None) == m.MOE_ERR_UNSUPPORTED_SHAPE
    assert L.fp8_quant_1x128(None, 4, 128, 100, None, None, None) == m.MOE_ERR_INVALID_ARG
    assert L.fp8_quant_1x128(None, 0, 128, 128, None, None, None) == m.MOE_OK  # empty: nothing enqueued
    assert L.fp8_quant_128x128(None, 100, 128, None, None, None) == m.MOE_ERR_UNSUPPORTED_SHAPE
    assert L.fp8_blockscaled_gemm(None, None, None, None, None, 4, 100, 128, None, None) == m.MOE_ERR_UNSUPPORTED_SHAPE
    assert L.fp8_blockscaled_gemm(None, None, None, None, None, 4, 128, 128, None, None) == m.MOE_ERR_INVALID_ARG
    bad = m.config(7168, 2000, 256, 8)
    assert m.moe_workspace_size(bad, 64) == 0
    import ctypes as C
    assert L.moe_forward(C.byref(bad), None, None, None, 64, None, 0, None, None, None, 0, None, None) == \
        m.MOE_ERR_UNSUPPORTED_SHAPE
    cfg = m.config(512, 256, 16, 4)
    assert L.moe_forward(C.byref(cfg), None, None, None, 64, None, 7, None, None, None, 0, None, None) == \
        m.MOE_ERR_INVALID_ARG
    # too many experts per token / groups that cannot hold top_k
    assert m.moe_workspace_size(m.config(512, 256, 16, 17), 8) == 0
    assert m.moe_workspace_size(m.config(512, 256, 16, 5, 1, 4, 1), 8) == 0
    # one expert per group: a group score (sum of the two best) is undefined
    assert m.moe_workspace_size(m.config(512, 256, 16, 4, 1, 16, 4), 8) == 0
    assert L.moe_forward(C.byref(m.config(512, 256, 16, 4, 1, 16, 4)), None, None, None, 64, None, 0, None, None,
                         None, 0, None, None) == m.MOE_ERR_UNSUPPORTED_SHAPE
    assert m.moe_workspace_size(m.config(512, 256, 16, 4, 1, 8, 4), 8) > 0
    # a valid call with non-null pointers reaches the device check
    assert L.fp8_quant_1x128(16, 4, 128, 128, 16, 16, None) == m.MOE_ERR_NO_DEVICE


def test_gemm_variant_switch(m):
    L = m.lib
    for v in (m.MOE_GEMM_SINGLE, m.MOE_GEMM_PAIR, m.MOE_GEMM_AUTO):
        assert L.moe_set_gemm_variant(v) == m.MOE_OK
    assert L.moe_set_gemm_variant(m.MOE_GEMM_TALL) == m.MOE_OK
    assert L.moe_set_gemm_variant(m.MOE_GEMM_AUTO) == m.MOE_OK
    assert L.moe_set_gemm_variant(3) == m.MOE_ERR_INVALID_ARG
    assert L.moe_set_gemm_variant(5) == m.MOE_ERR_INVALID_ARG
    assert L.moe_set_gemm_variant(-1) == m.MOE_ERR_INVALID_ARG


def test_gemm_kernel_choice(m):
    v3 = m.config(7168, 2048, 256, 8, 1, 8, 4)
    try:
        # AUTO: single CTAs at every size
        for T in (0, 64, 4096, 16384):
            assert m.moe_gemm_kernel_for(v3, T) == m.MOE_GEMM_SINGLE
        # hidden 7168 = 56 blocks pairs up; 640 = 5 blocks does not
        odd = m.config(640, 256, 16, 4, 1, 0, 0)
        m.moe_set_gemm_variant(m.MOE_GEMM_PAIR)
        assert m.moe_gemm_kernel_for(v3, 64) == m.MOE_GEMM_PAIR
        assert m.moe_gemm_kernel_for(odd, 64) == m.MOE_GEMM_SINGLE
        m.moe_set_gemm_variant(m.MOE_GEMM_TALL)
        assert m.moe_gemm_kernel_for(v3, 4096) == m.MOE_GEMM_TALL
        assert m.moe_gemm_kernel_for(odd, 4096) == m.MOE_GEMM_SINGLE
        m.moe_set_gemm_variant(m.MOE_GEMM_SINGLE)
        assert m.moe_gemm_kernel_for(v3, 16384) == m.MOE_GEMM_SINGLE
        pow2 = m.config(7168, 2048, 256, 8, 1, 8, 4, scale_mode=m.MOE_SCALE_POW2)
        assert m.moe_gemm_kernel_for(pow2, 16384) == m.MOE_GEMM_BLOCK_SCALED
        with pytest.raises(m.MoeError):
            m.moe_gemm_kernel_for(v3, -1)
    finally:
        m.moe_set_gemm_variant(m.MOE_GEMM_AUTO)


def test_contraction_and_alignment_limits_without_device(m):
    import ctypes as C
    L = m.lib
    # the GEMM kernels keep the scales of at most 256 K blocks per tile
    for H, I in [(32768, 2048), (7168, 32768)]:
        assert m.moe_workspace_size(m.config(H, I, 16, 4), 8) > 0
    for H, I in [(32768 + 128, 2048), (7168, 32768 + 128), (65536, 2048)]:
        assert m.moe_workspace_size(m.config(H, I, 16, 4), 8) == 0
    assert L.fp8_blockscaled_gemm(16, 16, 16, 16, 16, 4, 128, 32768 + 128, 16, None) == m.MOE_ERR_UNSUPPORTED_SHAPE
    # operands 16-byte aligned, scales and the error word 4-byte aligned
    assert L.fp8_blockscaled_gemm(16, 18, 16, 16, 16, 4, 128, 128, 16, None) == m.MOE_ERR_INVALID_ARG
    assert L.fp8_blockscaled_gemm(16, 16, 16, 17, 16, 4, 128, 128, 16, None) == m.MOE_ERR_INVALID_ARG
    assert L.fp8_blockscaled_gemm(16, 16, 16, 16, 16, 4, 128, 128, 18, None) == m.MOE_ERR_INVALID_ARG
    assert L.fp8_blockscaled_gemm(24, 16, 16, 16, 16, 4, 128, 128, 16, None) == m.MOE_ERR_INVALID_ARG
    assert L.fp8_blockscaled_gemm(16, 20, 16, 20, 16, 4, 128, 128, 20, None) == m.MOE_ERR_NO_DEVICE
    assert L.fp8_blockscaled_gemm(16, 16, 16, 16, 16, 4, 128, 32768, 16, None) == m.MOE_ERR_NO_DEVICE
    assert L.moe_bias_update(18, 16, 16, 64, C.c_float(0.001), None) == m.MOE_ERR_INVALID_ARG
    assert L.moe_bias_update(16, 16, 16, 64, C.c_float(0.001), None) == m.MOE_ERR_NO_DEVICE
    # moe_forward: misaligned weight scales are rejected before the device check
    cfg = m.config(512, 256, 16, 4)
    for s13, s2, bias in [(18, 16, 16), (16, 18, 16), (16, 16, 18)]:
        w = m._binding.MoeWeights(16, s13, 16, s2, 16)
        assert L.moe_forward(C.byref(cfg), C.byref(w), bias, 16, 64, 16, 0, None, None, 256, 1 << 40, 16, None) \
            == m.MOE_ERR_INVALID_ARG
    w = m._binding.MoeWeights(16, 16, 16, 16, 16)
    assert L.moe_forward(C.byref(cfg), C.byref(w), 16, 16, 64, 16, 0, None, None, 256, 1 << 40, 16, None) \
        == m.MOE_ERR_NO_DEVICE


def test_workspace_layout_is_disjoint_and_aligned(m):
    for (H, I, Nr, Kr, T) in [(512, 256, 16, 4, 256), (7168, 2048, 256, 8, 64), (7168, 2048, 256, 8, 4096),
                              (7168, 2048, 256, 8, 16384), (512, 256, 16, 4, 1)]:
        cfg = m.config(H, I, Nr, Kr)
        L = m.moe_workspace_layout(cfg, T)
        spans = sorted(v for k, v in L.items() if k != "total")
        for (o, n) in spans:
            assert o % 256 == 0
        for (o1, n1), (o2, _) in zip(spans, spans[1:]):
            assert o1 + n1 <= o2
        assert spans[-1][0] + spans[-1][1] <= L["total"] == m.moe_workspace_size(cfg, T)
        R = T * Kr
        assert L["ap"][1] == R * H and L["y"][1] == (R + T) * H * 4 and L["hq"][1] == (R + T) * I


def test_route_workspace_size(m):
    cfg = m.config(7168, 2048, 256, 8)
    assert m.moe_route_workspace_size(cfg, 4096) >= 4096 * 256 * 4
    assert m.moe_route_workspace_size(cfg, 0) >= 0


def test_seq_balance_loss_validation_without_device(m):
    import ctypes as C
    L = m.lib
    cfg = m.config(512, 256, 16, 4)
    big = 1 << 40
    a = C.c_float(1e-4)
    assert L.moe_seq_balance_loss(C.byref(cfg), 0, 8, a, None, 0, None, None, None) == m.MOE_OK
    assert L.moe_seq_balance_loss(C.byref(cfg), 96, 40, a, 256, big, 16, 16, None) == m.MOE_ERR_INVALID_ARG
    assert L.moe_seq_balance_loss(C.byref(cfg), 96, 0, a, 256, big, 16, 16, None) == m.MOE_ERR_INVALID_ARG
    assert L.moe_seq_balance_loss(C.byref(cfg), 96, 32, C.c_float(float("nan")), 256, big, 16, 16, None) == \
        m.MOE_ERR_INVALID_ARG
    assert L.moe_seq_balance_loss(C.byref(cfg), 96, 32, a, 128, big, 16, 16, None) == m.MOE_ERR_INVALID_ARG
    assert L.moe_seq_balance_loss(C.byref(cfg), 96, 32, a, 256, big, 18, 16, None) == m.MOE_ERR_INVALID_ARG
    assert L.moe_seq_balance_loss(C.byref(cfg), 96, 32, a, 256, 1024, 16, 16, None) == \
        m.MOE_ERR_WORKSPACE_TOO_SMALL
    assert L.moe_seq_balance_loss(C.byref(cfg), 96, 32, a, 256, big, 16, 16, None) == m.MOE_ERR_NO_DEVICE


def test_workspace_guard_bands_catch_overruns(m):
    """The guard bands the GPU tests put around every workspace and output
    buffer: intact after a call that stays inside, reported when a byte past
    either end changes (exercised here on host memory)."""
    import sys

    import torch
    layer = m.MoeLayer(dict(H=512, I=256, Nr=16, Kr=4, Ns=1), "cpu")
    layer.guard_bytes = 4096
    ws = layer.workspace(64)
    assert ws.numel() == m.moe_workspace_size(layer.cfg, 64)
    ws.fill_(0)              # the call's own bytes may change freely
    layer.check_guards()
    buf, g, n = layer._guarded[0]
    buf[g + n] = 0           # one byte past the end
    with pytest.raises(RuntimeError):
        layer.check_guards()
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from _moe_util import guarded_empty
    t, check = guarded_empty((3, 5), torch.float32, "cpu")
    t.fill_(1.0)
    check()
    raw = torch.tensor([], dtype=torch.uint8).set_(t.untyped_storage())
    raw[0] = 0               # first byte of the leading band
    with pytest.raises(AssertionError):
        check()


def test_expert_parallel_entry_points_validate_on_the_host(m):
    import ctypes as C
    L = m.lib
    cfg = m.config(512, 256, 16, 4)
    # packed row: H codes, H/128 scales, K_r slots and K_r gates, padded to 16 bytes
    assert m.moe_ep_row_bytes(cfg) == (512 + 4 * 4 + 8 * 4 + 15) // 16 * 16
    assert m.moe_ep_row_bytes(m.config(7168, 2048, 256, 8)) == 7168 + 224 + 64
    assert m.moe_ep_row_bytes(m.config(7168, 2000, 256, 8)) == 0        # invalid shape
    assert L.moe_ep_dispatch_workspace_size(C.byref(cfg), 3, 64) == 0    # 16 experts do not split over 3 ranks
    assert L.moe_ep_dispatch_workspace_size(C.byref(cfg), 4, 64) >= 256
    # world that does not divide the experts; too small a send capacity
    assert L.moe_ep_dispatch(C.byref(cfg), 3, 16, 16, 16, 16, 8, 16, 64, 16, 16, 16, None, 256, 1 << 20, 16,
                             None) == m.MOE_ERR_INVALID_ARG
    assert L.moe_ep_dispatch(C.byref(cfg), 4, 16, 16, 16, 16, 8, 16, 31, 16, 16, 16, None, 256, 1 << 20, 16,
                             None) == m.MOE_ERR_INVALID_ARG
    assert L.moe_ep_dispatch(C.byref(cfg), 4, 16, 16, 16, 16, 8, 16, 32, 16, 16, 16, None, 256, 1 << 20, 16,
                             None) == m.MOE_ERR_NO_DEVICE
    # the experts' side takes no shared expert and the layer's packed row only
    loc = m.config(512, 256, 4, 4, 0)
    rb = m.moe_ep_row_bytes(loc)
    w = m.MoeWeights(16, 16, 16, 16, None)
    assert L.moe_ep_experts(C.byref(m.config(512, 256, 4, 4, 1)), C.byref(w), 16, 8, rb, 16, 256, 1 << 30, 16,
                            None) == m.MOE_ERR_INVALID_ARG
    assert L.moe_ep_experts(C.byref(loc), C.byref(w), 16, 8, rb + 16, 16, 256, 1 << 30, 16, None) == \
        m.MOE_ERR_INVALID_ARG
    assert L.moe_ep_experts(C.byref(loc), C.byref(w), 16, 8, rb, 16, 256, 1 << 30, 16, None) == m.MOE_ERR_NO_DEVICE
    assert L.moe_ep_combine(C.byref(cfg), 0, 16, 8, 16, 16, None, 16, 0, None) == m.MOE_ERR_INVALID_ARG
    assert L.moe_ep_combine(C.byref(cfg), 2, 16, 8, 16, 16, None, 16, 0, None) == m.MOE_ERR_NO_DEVICE


def test_backward_entry_points_validate_on_the_host(m):
    import ctypes as C
    L = m.lib
    cfg = m.config(512, 256, 16, 4)
    assert L.moe_backward_workspace_size(C.byref(cfg), 64) > 0
    assert L.moe_backward_workspace_size(C.byref(m.config(512, 200, 16, 4)), 64) == 0
    w = m.MoeWeights(16, 16, 16, 16, 16)
    args = (16, 16, 16, 16, 16, 16, 64, 16, 16, 16, 256, 1 << 30, 256, 1 << 33, 16, None)
    pow2 = m.config(512, 256, 16, 4, scale_mode=m.MOE_SCALE_POW2)
    assert L.moe_backward(C.byref(pow2), C.byref(w), *args) == m.MOE_ERR_NOT_IMPLEMENTED
    assert L.moe_backward(C.byref(cfg), C.byref(w), *args[:6], 0, *args[7:]) == m.MOE_ERR_INVALID_ARG  # T = 0
    small = args[:11] + (1024,) + args[12:]   # forward workspace too small
    assert L.moe_backward(C.byref(cfg), C.byref(w), *small) == m.MOE_ERR_WORKSPACE_TOO_SMALL
    assert L.moe_backward(C.byref(cfg), C.byref(w), *args) == m.MOE_ERR_NO_DEVICE
    assert L.moe_transpose_weights(C.byref(cfg), C.byref(w), 16, 16, 16, 16, None) == m.MOE_ERR_NO_DEVICE


def test_profile_event_hook_validation(m):
    """The measurement hook takes the forward's 7 event handles, or 7 + 9 to
    also mark the backward's stages; a null handle among those it keeps is
    rejected; a null array turns it off.  (Handles are only stored here: no
    forward runs while the fake ones are set.)"""
    import ctypes as C
    L = m.lib
    nf, nb = m.MOE_PROFILE_EVENTS, m.MOE_PROFILE_BWD_EVENTS
    assert (nf, nb) == (7, 9)
    try:
        fake = (C.c_void_p * (nf + nb))(*range(1, nf + nb + 1))
        assert L.moe_profile_events(fake, nf) == m.MOE_OK
        assert L.moe_profile_events(fake, nf + nb) == m.MOE_OK
        assert L.moe_profile_events(fake, nf - 1) == m.MOE_ERR_INVALID_ARG
        holes = (C.c_void_p * (nf + nb))(*range(1, nf + nb + 1))
        holes[nf + 3] = None  # a backward handle missing: rejected when all 16 are given
        assert L.moe_profile_events(holes, nf + nb) == m.MOE_ERR_INVALID_ARG
        assert L.moe_profile_events(holes, nf) == m.MOE_OK  # forward-only: the hole is not kept
    finally:
        assert L.moe_profile_events(None, 0) == m.MOE_OK
