"""CPU oracle of the FP8 DeepSeekMoE layer forward -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It wraps ``moe_oracle.c`` (plain C,
double precision, built with gcc) through ctypes and adds the integer-only
steps (histogram, expert-contiguous order) and the sequence-wise balance loss
(a metric of the routing) in numpy.  It shares no code with
the CUDA library and never calls it.

Sources are cited in ``moe_oracle.c`` (page title and section); the short
names [P1]..[P4] used here refer to the same pages.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``moe_oracle.c`` into ``liboracle.so`` next to it (gcc, OpenMP,
    no fast-math, no FMA contraction)."""
    if not force and os.path.exists(_LIB_PATH) and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
           "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class Cfg(C.Structure):
    _fields_ = [("H", C.c_int32), ("I", C.c_int32), ("Nr", C.c_int32), ("Kr", C.c_int32),
                ("Ns", C.c_int32), ("n_groups", C.c_int32), ("topk_groups", C.c_int32),
                ("scale_mode", C.c_int32), ("route_scale", C.c_double)]

# scale modes of the quantizers: S = amax/448 (the pages' recipe), or the
# power-of-two variant (S = the smallest 2^e with amax <= 448 * 2^e)
SCALE_AMAX = 0
SCALE_POW2 = 1


def _p(a: np.ndarray):
    return a.ctypes.data_as(C.c_void_p)


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = C.CDLL(_LIB_PATH)
            vp, i64, f32 = C.c_void_p, C.c_int64, C.c_float
            L.moe_oracle_e4m3_decode.argtypes = [C.c_uint8]
            L.moe_oracle_e4m3_decode.restype = C.c_double
            L.moe_oracle_e4m3_encode.argtypes = [C.c_float]
            L.moe_oracle_e4m3_encode.restype = C.c_uint8
            L.moe_oracle_quant_1x128_bf16.argtypes = [vp, i64, i64, i64, vp, vp, C.c_int]
            L.moe_oracle_quant_1x128_f32.argtypes = [vp, i64, i64, vp, vp, C.c_int]
            L.moe_oracle_quant_128x128.argtypes = [vp, i64, i64, vp, vp, C.c_int]
            L.moe_oracle_blockscaled_gemm.argtypes = [vp, vp, vp, vp, i64, i64, i64, vp]
            L.moe_oracle_route.argtypes = [C.POINTER(Cfg), vp, i64, vp, vp, vp, vp, vp, vp]
            L.moe_oracle_expert_ffn.argtypes = [C.POINTER(Cfg), vp, vp, i64, vp, vp, vp, vp, vp, vp, vp, vp]
            L.moe_oracle_forward.argtypes = [C.POINTER(Cfg), vp, vp, i64, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
            L.moe_oracle_forward.restype = C.c_int
            L.moe_oracle_bias_update.argtypes = [vp, vp, C.c_int, i64, f32]
            L.moe_oracle_round_bf16.argtypes = [vp, i64, vp]
            L.moe_oracle_num_threads.restype = C.c_int
            L.moe_oracle_set_num_threads.argtypes = [C.c_int]
            _lib = L
    return _lib


def num_threads() -> int:
    return int(lib().moe_oracle_num_threads())


def set_num_threads(n: int) -> None:
    """Threads of the oracle's later parallel loops (OpenMP), from this thread."""
    lib().moe_oracle_set_num_threads(int(n))


def cfg(H, I, Nr, Kr, Ns=1, n_groups=0, topk_groups=0, route_scale=1.0, scale_mode=SCALE_AMAX) -> Cfg:
    # group-limited routing scores a group by the sum of its two best biased
    # scores, which needs at least two experts per group
    assert n_groups == 0 or (Nr % n_groups == 0 and Nr // n_groups >= 2), "groups need two experts or more"
    return Cfg(H, I, Nr, Kr, Ns, n_groups, topk_groups, scale_mode, route_scale)


def _f32(a) -> np.ndarray:
    """float32 numpy copy of a numpy array or a (possibly device) torch tensor."""
    if not isinstance(a, np.ndarray) and hasattr(a, "detach"):
        a = a.detach().cpu().float().numpy()
    return np.ascontiguousarray(a, dtype=np.float32)


def _u16(a) -> np.ndarray:
    """bf16 data as its raw 16-bit patterns (accepts a torch bf16 tensor or a
    uint16 numpy array)."""
    if isinstance(a, np.ndarray):
        assert a.dtype == np.uint16
        return np.ascontiguousarray(a)
    import torch
    assert a.dtype == torch.bfloat16
    return np.ascontiguousarray(a.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


# ------------------------------------------------------------------ E4M3
def e4m3_decode(code: int) -> float:
    return float(lib().moe_oracle_e4m3_decode(int(code)))


def e4m3_encode(v: float) -> int:
    return int(lib().moe_oracle_e4m3_encode(float(v)))


def e4m3_decode_table() -> np.ndarray:
    return np.array([e4m3_decode(c) for c in range(256)], dtype=np.float64)


# ------------------------------------------------------------- quantizers
def quant_1x128(x, mode: int = SCALE_AMAX) -> tuple[np.ndarray, np.ndarray]:
    """1x128 activation quantizer: x bf16 [rows, cols] -> (codes u8 [rows,
    cols], scales f32 [rows, cols/128])."""
    xu = _u16(x)
    rows, cols = xu.shape
    assert cols % 128 == 0
    q = np.empty((rows, cols), np.uint8)
    s = np.empty((rows, cols // 128), np.float32)
    lib().moe_oracle_quant_1x128_bf16(_p(xu), rows, cols, cols, _p(q), _p(s), int(mode))
    return q, s


def quant_1x128_f32(x: np.ndarray, mode: int = SCALE_AMAX) -> tuple[np.ndarray, np.ndarray]:
    x = np.ascontiguousarray(x, dtype=np.float32)
    rows, cols = x.shape
    q = np.empty((rows, cols), np.uint8)
    s = np.empty((rows, cols // 128), np.float32)
    lib().moe_oracle_quant_1x128_f32(_p(x), rows, cols, _p(q), _p(s), int(mode))
    return q, s


def quant_128x128(w, mode: int = SCALE_AMAX) -> tuple[np.ndarray, np.ndarray]:
    """128x128 weight quantizer: w bf16 [n, k] -> (codes [n, k], scales f32
    [n/128, k/128])."""
    wu = _u16(w)
    n, k = wu.shape
    assert n % 128 == 0 and k % 128 == 0
    q = np.empty((n, k), np.uint8)
    s = np.empty((n // 128, k // 128), np.float32)
    lib().moe_oracle_quant_128x128(_p(wu), n, k, _p(q), _p(s), int(mode))
    return q, s


def dequant(q: np.ndarray, s: np.ndarray, block_rows: int) -> np.ndarray:
    """Dequantize codes with scales tiled as (block_rows x 128)."""
    dec = e4m3_decode_table()[q]
    sf = np.repeat(np.repeat(s.astype(np.float64), block_rows, axis=0), 128, axis=1)
    return dec * sf


# ------------------------------------------------------------------ GEMM
def blockscaled_gemm(A, sA, B, sB) -> np.ndarray:
    """C = A x B^T with 1x128 scales on A [M,K] and 128x128 scales on B [N,K],
    promotion every 128 K; double result [M, N]."""
    A = np.ascontiguousarray(A, np.uint8)
    B = np.ascontiguousarray(B, np.uint8)
    sA = np.ascontiguousarray(sA, np.float32)
    sB = np.ascontiguousarray(sB, np.float32)
    M, K = A.shape
    N = B.shape[0]
    assert B.shape[1] == K and K % 128 == 0 and N % 128 == 0
    Cm = np.empty((M, N), np.float64)
    lib().moe_oracle_blockscaled_gemm(_p(A), _p(sA), _p(B), _p(sB), M, N, K, _p(Cm))
    return Cm


# --------------------------------------------------------------- routing
def route(cf: Cfg, x, Wr, bias, want_s: bool = False):
    """Returns (idx i32 [T,Kr], gate f64 [T,Kr], gap f32 [T], s f64 [T,Nr] or None)."""
    xu = _u16(x)
    wu = _u16(Wr)
    b = _f32(bias)
    T = xu.shape[0]
    idx = np.empty((T, cf.Kr), np.int32)
    gate = np.empty((T, cf.Kr), np.float64)
    gap = np.empty((T,), np.float32)
    s = np.empty((T, cf.Nr), np.float64) if want_s else None
    lib().moe_oracle_route(C.byref(cf), _p(xu), T, _p(wu), _p(b), _p(idx), _p(gate), _p(gap),
                           _p(s) if want_s else None)
    return idx, gate, gap, s


def histogram(idx: np.ndarray, Nr: int) -> np.ndarray:
    """Per-expert number of (token, slot) assignments."""
    return np.bincount(np.asarray(idx).reshape(-1), minlength=Nr).astype(np.int32)


def expert_order(idx: np.ndarray, Nr: int):
    """Expert-contiguous order of the (token, slot) assignments: stable
    counting sort by expert id, ties by token then slot (row-major order of
    idx).  Returns (offsets [Nr+1], src_flat [T*Kr]) where src_flat[p] is the
    row-major (t*Kr + k) assignment placed at position p."""
    flat = np.asarray(idx).reshape(-1)
    order = np.argsort(flat, kind="stable")
    counts = np.bincount(flat, minlength=Nr)
    offsets = np.zeros(Nr + 1, np.int64)
    offsets[1:] = np.cumsum(counts)
    return offsets, order.astype(np.int64)


def seq_balance_loss(s, idx, Nr: int, Kr: int, seq_len: int, alpha: float = 1e-4) -> np.ndarray:
    """Sequence-wise balance loss of each run of ``seq_len`` consecutive tokens.

    "DeepSeek-V3 Technischer Bericht", Methode section 2, names a small
    complementary sequence-wise balance loss with alpha = 0.0001 but prints no
    formula.  This follows the form the DeepSeek-V3 technical report gives it,
    for one sequence of L tokens:
        f_i  = N_r / (K_r L) * (number of tokens of the sequence that select expert i)
        P_i  = (1 / L) * sum_t s_{i,t} / sum_j s_{j,t}
        loss = alpha * sum_i f_i P_i
    where s_{i,t} are the sigmoid affinities of all N_r routed experts and the
    selection is the routing decision.  s: [T, Nr] doubles, idx: [T, Kr]
    expert ids; T must be a multiple of seq_len.  Returns one loss per
    sequence, in double precision.
    """
    s = np.asarray(s, np.float64)
    idx = np.asarray(idx)
    T = s.shape[0]
    assert s.shape == (T, Nr) and idx.shape == (T, Kr) and seq_len >= 1 and T % seq_len == 0
    L = seq_len
    out = np.empty(T // L, np.float64)
    for q in range(T // L):
        seq_s = s[q * L:(q + 1) * L]
        picks = np.zeros(Nr, np.float64)
        for row in idx[q * L:(q + 1) * L]:
            for e in row:
                picks[int(e)] += 1.0
        f = Nr / (Kr * L) * picks
        P = (seq_s / seq_s.sum(axis=1, keepdims=True)).sum(axis=0) / L
        out[q] = alpha * float(np.dot(f, P))
    return out


# ------------------------------------------------------------ expert FFN
def expert_ffn(cf: Cfg, xq, xs, W13q, s13, W2q, s2, want_h: bool = False):
    xq = np.ascontiguousarray(xq, np.uint8)
    xs = np.ascontiguousarray(xs, np.float32)
    n = xq.shape[0]
    y = np.empty((n, cf.H), np.float64)
    h = np.empty((n, cf.I), np.float32) if want_h else None
    hq = np.empty((n, cf.I), np.uint8) if want_h else None
    hs = np.empty((n, cf.I // 128), np.float32) if want_h else None
    arrs = [np.ascontiguousarray(a) for a in (W13q, s13, W2q, s2)]
    lib().moe_oracle_expert_ffn(C.byref(cf), _p(xq), _p(xs), n, *[_p(a) for a in arrs], _p(y),
                                _p(h) if want_h else None, _p(hq) if want_h else None,
                                _p(hs) if want_h else None)
    return (y, h, hq, hs) if want_h else y


# ----------------------------------------------------------- full layer
def forward(cf: Cfg, x, Wr, bias, experts, tokens=None):
    """Layer output for the listed tokens (all when None).

    experts: sequence of Nr+Ns tuples (W13q, s13, W2q, s2) of numpy arrays, or
    None for an expert that no listed token selects.
    Returns dict(out=f64 [n,H], out_bf16=u16 [n,H], idx, gate, gap)."""
    xu = _u16(x)
    T, H = xu.shape
    tok = np.arange(T, dtype=np.int64) if tokens is None else np.ascontiguousarray(tokens, np.int64)
    n = tok.shape[0]
    E = cf.Nr + cf.Ns
    assert len(experts) == E
    keep = []
    ptrs = [(C.c_void_p * E)() for _ in range(4)]
    for e, ex in enumerate(experts):
        if ex is None:
            for j in range(4):
                ptrs[j][e] = None
            continue
        arrs = [np.ascontiguousarray(a) for a in ex]
        keep.append(arrs)
        for j in range(4):
            ptrs[j][e] = arrs[j].ctypes.data
    wu = _u16(Wr)
    b = _f32(bias)
    out = np.empty((n, H), np.float64)
    outb = np.empty((n, H), np.uint16)
    idx = np.empty((n, cf.Kr), np.int32)
    gate = np.empty((n, cf.Kr), np.float64)
    gap = np.empty((n,), np.float32)
    rc = lib().moe_oracle_forward(C.byref(cf), _p(xu), _p(tok), n, _p(wu), _p(b), ptrs[0], ptrs[1], ptrs[2],
                                  ptrs[3], _p(out), _p(outb), _p(idx), _p(gate), _p(gap))
    if rc != 0:
        raise ValueError("oracle forward: an expert needed by a listed token was not supplied")
    return dict(out=out, out_bf16=outb, idx=idx, gate=gate, gap=gap)


def bias_update(bias, counts, Nr: int, total: int, gamma: float = 0.001) -> np.ndarray:
    b = np.array(bias, dtype=np.float32, copy=True)
    c = np.ascontiguousarray(counts, np.int32)
    lib().moe_oracle_bias_update(_p(b), _p(c), Nr, int(total), float(gamma))
    return b


def round_bf16(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, np.float64)
    o = np.empty(v.shape, np.uint16)
    lib().moe_oracle_round_bf16(_p(v), v.size, _p(o))
    return o
