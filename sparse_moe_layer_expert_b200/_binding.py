"""ctypes binding of libmoefp8.so (the C ABI declared in include/moe_fp8.h).

Argument marshalling only: tensors are passed as raw device pointers, outputs
are allocated with torch when the caller does not supply them, and every
status code is turned into an exception.  All arithmetic of the layer runs in
the library's CUDA kernels; there is no Python or CPU fallback.  If the
library is missing this module raises ImportError at import time.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoefp8.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python sparse_moe_layer_expert_b200/build.py`")

lib = C.CDLL(LIB_PATH)

MOE_OK = 0
MOE_ERR_INVALID_ARG = -1
MOE_ERR_UNSUPPORTED_SHAPE = -2
MOE_ERR_WORKSPACE_TOO_SMALL = -3
MOE_ERR_CUDA = -4
MOE_ERR_TIMEOUT = -5
MOE_ERR_NOT_IMPLEMENTED = -6
MOE_ERR_NO_DEVICE = -7
MOE_ERR_DEVICE = -8
MOE_DEVERR_TIMEOUT = 1
MOE_DEVERR_BAD_INDEX = 2
MOE_DTYPE_BF16 = 0
MOE_DTYPE_F32 = 1
MOE_SCALE_AMAX = 0  # S = amax / 448 (the pages)
MOE_SCALE_POW2 = 1  # power-of-two scales, applied by the tensor core

EXPORTS = (
    "moe_status_string", "moe_abi_version", "fp8_quant_1x128", "fp8_quant_128x128", "fp8_quant_1x128_pow2",
    "fp8_quant_128x128_pow2", "fp8_blockscaled_gemm",
    "moe_route_workspace_size", "moe_route", "moe_workspace_size", "moe_forward", "moe_workspace_layout",
    "moe_bias_update", "moe_check_device_error", "moe_selftest_wait_timeout", "moe_profile_events",
    "moe_route_noalloc", "moe_seq_balance_loss", "moe_set_gemm_variant", "moe_gemm_kernel_for",
    "moe_ep_row_bytes", "moe_ep_dispatch_workspace_size", "moe_ep_dispatch", "moe_ep_experts_workspace_size",
    "moe_ep_experts", "moe_ep_combine", "moe_transpose_weights", "moe_backward_workspace_size", "moe_backward",
    "moe_backward_workspace_layout",
)
MOE_GEMM_AUTO = 0
MOE_GEMM_SINGLE = 1
MOE_GEMM_PAIR = 2
MOE_GEMM_BLOCK_SCALED = 3
MOE_GEMM_TALL = 4
MOE_ROUTE_NOALLOC_SCRATCH_BYTES = 16 << 20
MOE_PROFILE_EVENTS = 7
MOE_PROFILE_BWD_EVENTS = 9
PROFILE_STAGES = ("quantize", "route", "group", "gemm_gate_up", "gemm_down", "combine")
PROFILE_BWD_STAGES = ("recompute_gate_up", "dh", "swiglu_bwd", "dx_rows", "dx_combine", "wgrad_operands",
                      "wgrad_w2", "wgrad_w13")


class MoeConfig(C.Structure):
    _fields_ = [("hidden", C.c_int32), ("inter", C.c_int32), ("n_routed", C.c_int32), ("top_k", C.c_int32),
                ("n_shared", C.c_int32), ("n_groups", C.c_int32), ("topk_groups", C.c_int32),
                ("route_scale", C.c_float), ("scale_mode", C.c_int32)]


class MoeWeights(C.Structure):
    _fields_ = [("w13_dev", C.c_void_p), ("s13_dev", C.c_void_p), ("w2_dev", C.c_void_p),
                ("s2_dev", C.c_void_p), ("wr_dev", C.c_void_p)]


_LAYOUT_FIELDS = ("xq", "xs", "idx", "gate", "counts", "offsets", "pos", "ap", "as", "row_gate", "row_src", "hq",
                  "hs", "y", "meta", "logits", "blk_hist", "blk_base", "chunks")


class MoeWsLayout(C.Structure):
    _fields_ = [(f, C.c_size_t * 2) for f in _LAYOUT_FIELDS] + [("total", C.c_size_t)]


_vp, _i64, _i32, _f32, _sz = C.c_void_p, C.c_int64, C.c_int32, C.c_float, C.c_size_t
_cfgp = C.POINTER(MoeConfig)
lib.moe_status_string.restype = C.c_char_p
lib.moe_status_string.argtypes = [C.c_int]
lib.moe_abi_version.restype = C.c_int
lib.fp8_quant_1x128.argtypes = [_vp, _i64, _i64, _i64, _vp, _vp, _vp]
lib.fp8_quant_128x128.argtypes = [_vp, _i64, _i64, _vp, _vp, _vp]
lib.fp8_quant_1x128_pow2.argtypes = lib.fp8_quant_1x128.argtypes
lib.fp8_quant_128x128_pow2.argtypes = lib.fp8_quant_128x128.argtypes
lib.fp8_blockscaled_gemm.argtypes = [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _vp]
lib.moe_route_workspace_size.restype = _sz
lib.moe_route_workspace_size.argtypes = [_cfgp, _i64]
lib.moe_route.argtypes = [_cfgp, _vp, _vp, _vp, _i64, _vp, _vp, _vp, _vp, _sz, _vp, _vp]
lib.moe_route_noalloc.argtypes = [_cfgp, _vp, _vp, _vp, _i64, _vp, _vp, _vp, _vp, _vp]
lib.moe_workspace_size.restype = _sz
lib.moe_workspace_size.argtypes = [_cfgp, _i64]
lib.moe_forward.argtypes = [_cfgp, C.POINTER(MoeWeights), _vp, _vp, _i64, _vp, _i32, _vp, _vp, _vp, _sz, _vp, _vp]
lib.moe_workspace_layout.argtypes = [_cfgp, _i64, C.POINTER(MoeWsLayout)]
lib.moe_bias_update.argtypes = [_vp, _vp, _i32, _i64, _f32, _vp]
lib.moe_seq_balance_loss.argtypes = [_cfgp, _i64, _i64, _f32, _vp, _sz, _vp, _vp, _vp]
lib.moe_check_device_error.argtypes = [_vp, C.POINTER(C.c_int32), _vp]
lib.moe_selftest_wait_timeout.argtypes = [_vp, _i64, _vp]
lib.moe_profile_events.argtypes = [C.POINTER(_vp), _i32]
lib.moe_set_gemm_variant.argtypes = [_i32]
lib.moe_gemm_kernel_for.argtypes = [_cfgp, _i64]
lib.moe_ep_row_bytes.restype = _i64
lib.moe_ep_row_bytes.argtypes = [_cfgp]
lib.moe_ep_dispatch_workspace_size.restype = _sz
lib.moe_ep_dispatch_workspace_size.argtypes = [_cfgp, _i32, _i64]
lib.moe_ep_dispatch.argtypes = [_cfgp, _i32, _vp, _vp, _vp, _vp, _i64, _vp, _i64, _vp, _vp, _vp, _vp, _vp, _sz, _vp,
                                _vp]
lib.moe_ep_experts_workspace_size.restype = _sz
lib.moe_ep_experts_workspace_size.argtypes = [_cfgp, _i64]
lib.moe_ep_experts.argtypes = [_cfgp, C.POINTER(MoeWeights), _vp, _i64, _i64, _vp, _vp, _sz, _vp, _vp]
lib.moe_ep_combine.argtypes = [_cfgp, _i32, _vp, _i64, _vp, _vp, _vp, _vp, _i32, _vp]
lib.moe_transpose_weights.argtypes = [_cfgp, C.POINTER(MoeWeights), _vp, _vp, _vp, _vp, _vp]
class MoeBwdLayout(C.Structure):
    _fields_ = [(f, C.c_size_t * 2) for f in ("gu", "dh", "gh", "dgu", "dx_rows", "seg")] + [("P", C.c_int64),
                                                                                          ("total", C.c_size_t)]


lib.moe_backward_workspace_layout.argtypes = [_cfgp, _i64, C.POINTER(MoeBwdLayout)]
lib.moe_backward_workspace_size.restype = _sz
lib.moe_backward_workspace_size.argtypes = [_cfgp, _i64]
lib.moe_backward.argtypes = [_cfgp, C.POINTER(MoeWeights), _vp, _vp, _vp, _vp, _vp, _vp, _i64, _vp, _vp, _vp, _vp,
                             _sz, _vp, _sz, _vp, _vp]
for _name in EXPORTS:
    if _name not in ("moe_status_string", "moe_route_workspace_size", "moe_workspace_size", "moe_ep_row_bytes",
                     "moe_ep_dispatch_workspace_size", "moe_ep_experts_workspace_size",
                     "moe_backward_workspace_size"):
        getattr(lib, _name).restype = C.c_int


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {lib.moe_status_string(status).decode()} (status {status})")


def _check(status: int, where: str) -> None:
    if status != MOE_OK:
        raise MoeError(status, where)


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def config(hidden, inter, n_routed, top_k, n_shared=1, n_groups=0, topk_groups=0, route_scale=1.0,
           scale_mode=MOE_SCALE_AMAX) -> MoeConfig:
    return MoeConfig(hidden, inter, n_routed, top_k, n_shared, n_groups, topk_groups, route_scale, scale_mode)


def config_from(d: dict) -> MoeConfig:
    return config(d["H"], d["I"], d["Nr"], d["Kr"], d.get("Ns", 1), d.get("n_groups", 0), d.get("topk_groups", 0),
                  d.get("route_scale", 1.0), d.get("scale_mode", MOE_SCALE_AMAX))


def new_err_flag(device="cuda") -> torch.Tensor:
    return torch.zeros(1, dtype=torch.int32, device=device)


# ------------------------------------------------------------------ calls
def fp8_quant_1x128(x: torch.Tensor, q=None, scales=None, stream=None, pow2: bool = False):
    rows, cols = x.shape
    ld = x.stride(0)
    assert x.stride(1) == 1 and x.dtype == torch.bfloat16
    q = torch.empty((rows, cols), dtype=torch.uint8, device=x.device) if q is None else q
    scales = torch.empty((rows, cols // 128), dtype=torch.float32, device=x.device) if scales is None else scales
    fn = lib.fp8_quant_1x128_pow2 if pow2 else lib.fp8_quant_1x128
    _check(fn(_ptr(x), rows, cols, ld, _ptr(q), _ptr(scales), _stream(stream)), "fp8_quant_1x128")
    return q, scales


def fp8_quant_128x128(w: torch.Tensor, q=None, scales=None, stream=None, pow2: bool = False):
    assert w.is_contiguous() and w.dtype == torch.bfloat16
    n, k = w.shape[-2] * (w.numel() // (w.shape[-2] * w.shape[-1])), w.shape[-1]
    q = torch.empty(w.shape, dtype=torch.uint8, device=w.device) if q is None else q
    if scales is None:
        scales = torch.empty(w.shape[:-2] + (w.shape[-2] // 128, k // 128), dtype=torch.float32, device=w.device)
    fn = lib.fp8_quant_128x128_pow2 if pow2 else lib.fp8_quant_128x128
    _check(fn(_ptr(w), n, k, _ptr(q), _ptr(scales), _stream(stream)), "fp8_quant_128x128")
    return q, scales


def fp8_blockscaled_gemm(A, sA, B, sB, C=None, err=None, stream=None):
    M, K = A.shape
    N = B.shape[0]
    C = torch.empty((M, N), dtype=torch.bfloat16, device=A.device) if C is None else C
    err = new_err_flag(A.device) if err is None else err
    _check(lib.fp8_blockscaled_gemm(_ptr(A), _ptr(sA), _ptr(B), _ptr(sB), _ptr(C), M, N, K, _ptr(err),
                                    _stream(stream)), "fp8_blockscaled_gemm")
    return C


def moe_route_workspace_size(cfg: MoeConfig, T: int) -> int:
    return int(lib.moe_route_workspace_size(C.byref(cfg), T))


def moe_route(cfg: MoeConfig, x, wr, bias, idx=None, gate=None, counts=None, ws=None, err=None, stream=None):
    T = x.shape[0]
    dev = x.device
    idx = torch.empty((T, cfg.top_k), dtype=torch.int32, device=dev) if idx is None else idx
    gate = torch.empty((T, cfg.top_k), dtype=torch.float32, device=dev) if gate is None else gate
    counts = torch.empty((cfg.n_routed,), dtype=torch.int32, device=dev) if counts is None else counts
    if ws is None:
        ws = torch.empty(max(moe_route_workspace_size(cfg, T), 256), dtype=torch.uint8, device=dev)
    err = new_err_flag(dev) if err is None else err
    _check(lib.moe_route(C.byref(cfg), _ptr(x), _ptr(wr), _ptr(bias), T, _ptr(idx), _ptr(gate), _ptr(counts),
                         _ptr(ws), ws.numel(), _ptr(err), _stream(stream)), "moe_route")
    return idx, gate, counts


def moe_route_noalloc(cfg: MoeConfig, x, wr, bias, idx, gate, counts, err, stream=None):
    """moe_route with the library's fixed scratch; outputs must be supplied
    (this call is for callers that allocate nothing on the call path)."""
    _check(lib.moe_route_noalloc(C.byref(cfg), _ptr(x), _ptr(wr), _ptr(bias), x.shape[0], _ptr(idx), _ptr(gate),
                                 _ptr(counts), _ptr(err), _stream(stream)), "moe_route_noalloc")
    return idx, gate, counts


def moe_workspace_size(cfg: MoeConfig, T: int) -> int:
    return int(lib.moe_workspace_size(C.byref(cfg), T))


def moe_workspace_layout(cfg: MoeConfig, T: int) -> dict:
    L = MoeWsLayout()
    _check(lib.moe_workspace_layout(C.byref(cfg), T, C.byref(L)), "moe_workspace_layout")
    d = {f: (int(getattr(L, f)[0]), int(getattr(L, f)[1])) for f in _LAYOUT_FIELDS}
    d["total"] = int(L.total)
    return d


def weights_struct(w: dict) -> MoeWeights:
    return MoeWeights(_ptr(w["w13"]), _ptr(w["s13"]), _ptr(w["w2"]), _ptr(w["s2"]), _ptr(w["wr"]))


def moe_forward(cfg: MoeConfig, w: dict, bias, x, out=None, out_dtype=MOE_DTYPE_BF16, idx_out=None,
                counts_out=None, ws=None, err=None, stream=None):
    """w: dict with w13 u8 [E,2I,H], s13 f32 [E,2I/128,H/128], w2 u8 [E,H,I],
    s2 f32 [E,H/128,I/128], wr bf16 [Nr,H]."""
    T, H = x.shape
    dev = x.device
    if out is None:
        out = torch.empty((T, H), dtype=torch.float32 if out_dtype == MOE_DTYPE_F32 else torch.bfloat16, device=dev)
    if ws is None:
        ws = torch.empty(max(moe_workspace_size(cfg, T), 256), dtype=torch.uint8, device=dev)
    err = new_err_flag(dev) if err is None else err
    ws_struct = weights_struct(w)
    _check(lib.moe_forward(C.byref(cfg), C.byref(ws_struct), _ptr(bias), _ptr(x), T, _ptr(out), out_dtype,
                           _ptr(idx_out), _ptr(counts_out), _ptr(ws), ws.numel(), _ptr(err), _stream(stream)),
           "moe_forward")
    return out


def moe_bias_update(bias, counts, n_routed: int, total: int, gamma: float = 0.001, stream=None):
    _check(lib.moe_bias_update(_ptr(bias), _ptr(counts), n_routed, total, gamma, _stream(stream)), "moe_bias_update")
    return bias


def moe_seq_balance_loss(cfg: MoeConfig, T: int, seq_len: int, ws, err, loss=None, alpha: float = 1e-4,
                         stream=None):
    """Sequence-wise balance loss of each run of seq_len tokens of the batch
    the last moe_forward on `ws` routed (float32 [T // seq_len])."""
    loss = torch.empty(max(T // max(seq_len, 1), 1), dtype=torch.float32, device=ws.device) if loss is None else loss
    _check(lib.moe_seq_balance_loss(C.byref(cfg), T, seq_len, alpha, _ptr(ws), ws.numel(), _ptr(loss), _ptr(err),
                                    _stream(stream)), "moe_seq_balance_loss")
    return loss[:T // max(seq_len, 1)]


def moe_check_device_error(err, stream=None) -> tuple[int, int]:
    v = C.c_int32(0)
    st = lib.moe_check_device_error(_ptr(err), C.byref(v), _stream(stream))
    return st, int(v.value)


def moe_selftest_wait_timeout(err, limit_us: int, stream=None) -> None:
    _check(lib.moe_selftest_wait_timeout(_ptr(err), limit_us, _stream(stream)), "moe_selftest_wait_timeout")


def moe_profile_events(events) -> None:
    """events: MOE_PROFILE_EVENTS torch.cuda.Event(enable_timing=True), or
    None to stop recording."""
    if events is None:
        _check(lib.moe_profile_events(None, 0), "moe_profile_events")
        return
    arr = (_vp * len(events))(*[ev.cuda_event for ev in events])
    _check(lib.moe_profile_events(arr, len(events)), "moe_profile_events")


def moe_set_gemm_variant(variant: int) -> None:
    """Kernel choice of the grouped expert GEMMs (MOE_GEMM_AUTO, _SINGLE,
    _PAIR, _TALL), process-wide."""
    _check(lib.moe_set_gemm_variant(variant), "moe_set_gemm_variant")


def moe_gemm_kernel_for(cfg, T: int) -> int:
    """The grouped-GEMM kernel (MOE_GEMM_SINGLE, _PAIR, _TALL or _BLOCK_SCALED) the
    next moe_forward of T tokens runs under the current variant setting."""
    r = lib.moe_gemm_kernel_for(C.byref(cfg), int(T))
    if r < 0:
        _check(r, "moe_gemm_kernel_for")
    return r


# ---------------------------------------------------- expert parallelism
def moe_ep_row_bytes(cfg: MoeConfig) -> int:
    return int(lib.moe_ep_row_bytes(C.byref(cfg)))


def moe_ep_dispatch(cfg: MoeConfig, world: int, xq, xs, idx, gate, send_rows, send_counts, send_offsets, row_of,
                    self_rows=None, ws=None, err=None, stream=None):
    T = xq.shape[0]
    dev = xq.device
    if ws is None:
        ws = torch.empty(max(int(lib.moe_ep_dispatch_workspace_size(C.byref(cfg), world, T)), 256), dtype=torch.uint8,
                         device=dev)
    err = new_err_flag(dev) if err is None else err
    _check(lib.moe_ep_dispatch(C.byref(cfg), world, _ptr(xq), _ptr(xs), _ptr(idx), _ptr(gate), T, _ptr(send_rows),
                               send_rows.shape[0], _ptr(send_counts), _ptr(send_offsets), _ptr(row_of),
                               _ptr(self_rows), _ptr(ws), ws.numel(), _ptr(err), _stream(stream)), "moe_ep_dispatch")


def moe_ep_experts(cfg_local: MoeConfig, w_local: dict, rows, partial_out, ws=None, err=None, stream=None):
    n = rows.shape[0]
    dev = rows.device
    if ws is None:
        ws = torch.empty(max(int(lib.moe_ep_experts_workspace_size(C.byref(cfg_local), n)), 256), dtype=torch.uint8,
                         device=dev)
    err = new_err_flag(dev) if err is None else err
    wst = MoeWeights(_ptr(w_local["w13"]), _ptr(w_local["s13"]), _ptr(w_local["w2"]), _ptr(w_local["s2"]), None)
    _check(lib.moe_ep_experts(C.byref(cfg_local), C.byref(wst), _ptr(rows), n, rows.shape[1] if n else
                              moe_ep_row_bytes(cfg_local), _ptr(partial_out), _ptr(ws), ws.numel(), _ptr(err),
                              _stream(stream)), "moe_ep_experts")
    return partial_out


def moe_ep_combine(cfg: MoeConfig, world: int, x, row_of, back, y_shared, out, out_dtype=MOE_DTYPE_BF16, stream=None):
    _check(lib.moe_ep_combine(C.byref(cfg), world, _ptr(x), x.shape[0], _ptr(row_of), _ptr(back), _ptr(y_shared),
                              _ptr(out), out_dtype, _stream(stream)), "moe_ep_combine")
    return out


# ------------------------------------------------------------ backward
def moe_transpose_weights(cfg: MoeConfig, w: dict, stream=None) -> dict:
    """The dgrad GEMMs' weights: each expert's codes and block scales
    transposed (w13t [E, H, 2I], s13t, w2t [E, I, H], s2t)."""
    E, I2, H = w["w13"].shape
    I = I2 // 2
    dev = w["w13"].device
    t = dict(w13t=torch.empty((E, H, I2), dtype=torch.uint8, device=dev),
             s13t=torch.empty((E, H // 128, I2 // 128), dtype=torch.float32, device=dev),
             w2t=torch.empty((E, I, H), dtype=torch.uint8, device=dev),
             s2t=torch.empty((E, I // 128, H // 128), dtype=torch.float32, device=dev))
    ws = weights_struct(w)
    _check(lib.moe_transpose_weights(C.byref(cfg), C.byref(ws), _ptr(t["w13t"]), _ptr(t["s13t"]), _ptr(t["w2t"]),
                                     _ptr(t["s2t"]), _stream(stream)), "moe_transpose_weights")
    return t


def ctypes_cfg(cfg: MoeConfig):
    return C.byref(cfg)


def moe_backward_workspace_layout(cfg: MoeConfig, T: int) -> dict:
    L = MoeBwdLayout()
    _check(lib.moe_backward_workspace_layout(C.byref(cfg), T, C.byref(L)), "moe_backward_workspace_layout")
    d = {f: (int(getattr(L, f)[0]), int(getattr(L, f)[1])) for f in ("gu", "dh", "gh", "dgu", "dx_rows", "seg")}
    d["P"], d["total"] = int(L.P), int(L.total)
    return d


def moe_backward(cfg: MoeConfig, w: dict, wt: dict, x, dout, fwd_ws, dx=None, dW13=None, dW2=None, ws=None,
                 err=None, stream=None):
    """Gradients of the layer's expert FFNs (routing held fixed) for the batch
    whose forward left its state in fwd_ws: dx [T, H], dW13 [E, 2I, H],
    dW2 [E, H, I], all float32."""
    T, H = x.shape
    dev = x.device
    E, I2, _ = w["w13"].shape
    dx = torch.empty((T, H), dtype=torch.float32, device=dev) if dx is None else dx
    dW13 = torch.empty((E, I2, H), dtype=torch.float32, device=dev) if dW13 is None else dW13
    dW2 = torch.empty((E, H, I2 // 2), dtype=torch.float32, device=dev) if dW2 is None else dW2
    if ws is None:
        ws = torch.empty(max(int(lib.moe_backward_workspace_size(C.byref(cfg), T)), 256), dtype=torch.uint8,
                         device=dev)
    err = new_err_flag(dev) if err is None else err
    wst = weights_struct(w)
    _check(lib.moe_backward(C.byref(cfg), C.byref(wst), _ptr(wt["w13t"]), _ptr(wt["s13t"]), _ptr(wt["w2t"]),
                            _ptr(wt["s2t"]), _ptr(x), _ptr(dout), T, _ptr(dx), _ptr(dW13), _ptr(dW2), _ptr(fwd_ws),
                            fwd_ws.numel(), _ptr(ws), ws.numel(), _ptr(err), _stream(stream)), "moe_backward")
    return dx, dW13, dW2


def ws_view(ws: torch.Tensor, layout: dict, name: str, dtype, shape) -> torch.Tensor:
    """A typed view of one intermediate inside a moe_forward workspace."""
    off, nbytes = layout[name]
    esz = torch.empty((), dtype=dtype).element_size()
    n = 1
    for s in shape:
        n *= s
    assert n * esz <= nbytes
    return ws[off:off + n * esz].view(dtype).view(shape)
