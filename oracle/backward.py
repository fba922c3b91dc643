"""CPU oracle of the backward pass of one FP8 expert FFN -- TEST INFRASTRUCTURE ONLY.

Like the rest of ``oracle/``, only tests may import this module; it shares no
code with the CUDA library.  Double precision; the FP8 steps use the oracle's
own quantizers and E4M3 decode (``moe_oracle.c``).

What the pages fix: "DeepSeek-V3 Technischer Bericht" (xyznot.com/de),
Kernideen, FP8 bullet -- E4M3 for all tensors, 1x128 activation tiles,
128x128 weight blocks, FP32 accumulation promoted every N_c = 128 steps.  They
say nothing about the backward pass beyond "all tensors", so the tile
orientation is a reading (the DeepSeek-V3 technical report's recipe):

* every GEMM input is quantized along that GEMM's contraction dimension:
  - dgrad (contraction over the layer's output channels): the incoming
    gradient as 1x128 tiles along its row, the weights as the forward's
    128x128 blocks, transposed;
  - wgrad (contraction over tokens): both operands as 128x1 tiles, 128
    consecutive tokens of one channel (a ragged last tile holds fewer);
* every GEMM accumulates in FP32 per 128-long block, promoted into an FP32
  result (here: exact per-block sums, scaled and added in double, rounded to
  FP32 once at the end, as in the forward oracle);
* the SwiGLU backward is elementwise in double from the forward's FP32 G, U,
  rounded to FP32.

For one expert with input x [rows, H] (bf16), weights W1, W3 [I, H] and
W2 [H, I] (E4M3 codes with 128x128 block scales), the layer-output gradient
D of its rows [rows, H] (bf16) and the rows' gates g (1 for the shared
expert), the expert's output gradient is dY = g D:
    G = x W1^T, U = x W3^T, h = silu(G) * U, Y = h W2^T       (forward)
    dh  = g (D W2)                 dW2 = D^T (g h)
    dG  = dh * U * silu'(G)        dU  = dh * silu(G)
    dx  = dG W1 + dU W3            dW1 = dG^T x,   dW3 = dU^T x
with silu(G) = G sigma(G) and silu'(G) = sigma(G) (1 + G (1 - sigma(G))).
Where the gate sits is a reading.  For the dgrad, 1x128 tiles of g D along H
have the codes of D's tiles (g cancels in x / (amax / 448)), so D is
quantized and g scales the FP32 product: the exact-arithmetic result of
quantizing g D, without the rounding of g D deciding codes.  For the wgrad
(128x1 tiles along tokens, different gates in one tile) g rides on h, an
FP32 intermediate already: D^T (g h) = (g D)^T h.
The gate's own gradient (router backward) is not part of this.
"""
from __future__ import annotations

import numpy as np

from . import (SCALE_AMAX, _u16, blockscaled_gemm, e4m3_decode_table, quant_1x128, quant_1x128_f32, route)


def _pad_rows(a: np.ndarray, mult: int = 128) -> np.ndarray:
    r = a.shape[0]
    pad = (-r) % mult
    if pad == 0:
        return a
    return np.concatenate([a, np.zeros((pad,) + a.shape[1:], a.dtype)], axis=0)


def quant_128x1_bf16(x, mode: int = SCALE_AMAX) -> tuple[np.ndarray, np.ndarray]:
    """128x1 tiles of a bf16 matrix [rows, cols]: one scale per 128
    consecutive rows of one column (the last tile may be shorter).  Returns
    codes [rows, cols] and scales [ceil(rows/128), cols]."""
    xu = _u16(x)
    rows = xu.shape[0]
    q_t, s_t = quant_1x128(np.ascontiguousarray(_pad_rows(xu).T), mode)
    return np.ascontiguousarray(q_t.T[:rows]), np.ascontiguousarray(s_t.T)


def quant_128x1_f32(x: np.ndarray, mode: int = SCALE_AMAX) -> tuple[np.ndarray, np.ndarray]:
    """As quant_128x1_bf16 for FP32 values."""
    x = np.ascontiguousarray(x, np.float32)
    rows = x.shape[0]
    q_t, s_t = quant_1x128_f32(np.ascontiguousarray(_pad_rows(x).T), mode)
    return np.ascontiguousarray(q_t.T[:rows]), np.ascontiguousarray(s_t.T)


def rows_scaled_gemm(qa, sa, qb, sb) -> np.ndarray:
    """C[m, n] = sum_kb sa[m, kb] sb[n, kb] sum_{k in kb} dec(qa[m, k]) dec(qb[n, k])
    with one scale per row and 128-long K block on BOTH operands (the wgrad
    form, where K runs over tokens).  K is padded with zero codes to a
    multiple of 128.  Each block's sum of E4M3 products is exact in double;
    the result is double."""
    dec = e4m3_decode_table()
    A = dec[_pad_rows(np.asarray(qa).T).T]
    B = dec[_pad_rows(np.asarray(qb).T).T]
    sa = np.asarray(sa, np.float64)
    sb = np.asarray(sb, np.float64)
    M, K = A.shape
    N = B.shape[0]
    assert B.shape[1] == K and sa.shape == (M, K // 128) and sb.shape == (N, K // 128)
    out = np.zeros((M, N), np.float64)
    for kb in range(K // 128):
        P = A[:, kb * 128:(kb + 1) * 128] @ B[:, kb * 128:(kb + 1) * 128].T
        out += np.outer(sa[:, kb], sb[:, kb]) * P
    return out


def _f32(v: np.ndarray) -> np.ndarray:
    return np.asarray(v, np.float64).astype(np.float32).astype(np.float64)


def _as_f32_values(a) -> np.ndarray:
    """float32 values of a bf16 tensor, uint16 bf16 bit patterns or a float32
    array (bf16 -> float32 is exact, so quantizing either gives the same codes)."""
    if isinstance(a, np.ndarray) and a.dtype == np.float32:
        return np.ascontiguousarray(a)
    u = _u16(a).astype(np.uint32) << 16
    return np.ascontiguousarray(u.view(np.float32))


def expert_backward(x, dy, W13q, s13, W2q, s2, gate=None, mode: int = SCALE_AMAX) -> dict:
    """Backward of one expert FFN under the FP8 recipe above.

    x: bf16 [rows, H] (torch bf16 tensor or uint16 bit patterns); dy: the
    layer-output gradient D of the rows [rows, H], bf16 as x or float32
    values; gate: the rows' gates (double, [rows]) or None for 1;
    W13q u8 [2I, H] (gate rows 0..I-1, up rows I..2I-1), s13 f32 [2I/128, H/128];
    W2q u8 [H, I], s2 f32 [H/128, I/128].
    Returns FP32-rounded values (as float64 arrays): dx [rows, H],
    dW13 [2I, H], dW2 [H, I], the intermediates dh, dG, dU [rows, I], the
    forward's G, U, h [rows, I] and the wgrad operand gh = g h."""
    W13q = np.asarray(W13q, np.uint8)
    W2q = np.asarray(W2q, np.uint8)
    s13 = np.asarray(s13, np.float32)
    s2 = np.asarray(s2, np.float32)
    I2, H = W13q.shape
    I = I2 // 2
    dy = _as_f32_values(dy)
    g = np.ones(dy.shape[0]) if gate is None else np.asarray(gate, np.float64).reshape(-1)
    assert g.shape[0] == dy.shape[0]
    # forward recomputation (as the forward oracle: 1x128 x, FP32 G and U)
    xq, xs = quant_1x128(x, mode)
    G = _f32(blockscaled_gemm(xq, xs, W13q[:I], s13[:I // 128]))
    U = _f32(blockscaled_gemm(xq, xs, W13q[I:], s13[I // 128:]))
    sig = 1.0 / (1.0 + np.exp(-G))
    silu = G * sig
    h = _f32(silu * U)
    # dgrad of the down projection: D 1x128 along H, W2^T as [I, H] blocks,
    # the gate on the FP32 result
    dyq, dys = quant_1x128_f32(dy, mode)
    dh = _f32(g[:, None] * blockscaled_gemm(dyq, dys, np.ascontiguousarray(W2q.T), np.ascontiguousarray(s2.T)))
    # wgrad of the down projection: D and g h as 128x1 tiles along tokens
    gh = _f32(g[:, None] * h)
    dyq_c, dys_c = quant_128x1_f32(dy, mode)
    hq_c, hs_c = quant_128x1_f32(gh, mode)
    dW2 = _f32(rows_scaled_gemm(dyq_c.T, dys_c.T, hq_c.T, hs_c.T))
    # SwiGLU backward (double, rounded to FP32)
    dG = _f32(dh * U * sig * (1.0 + G * (1.0 - sig)))
    dU = _f32(dh * silu)
    # dgrad of gate/up: dG, dU 1x128 along I; W1^T, W3^T as [H, I] blocks;
    # one FP32 result over the whole 2I contraction
    dGq, dGs = quant_1x128_f32(dG, mode)
    dUq, dUs = quant_1x128_f32(dU, mode)
    dx = _f32(blockscaled_gemm(dGq, dGs, np.ascontiguousarray(W13q[:I].T), np.ascontiguousarray(s13[:I // 128].T))
              + blockscaled_gemm(dUq, dUs, np.ascontiguousarray(W13q[I:].T),
                                 np.ascontiguousarray(s13[I // 128:].T)))
    # wgrad of gate/up: dG, dU and x as 128x1 tiles along tokens
    xq_c, xs_c = quant_128x1_bf16(x, mode)
    dGq_c, dGs_c = quant_128x1_f32(dG, mode)
    dUq_c, dUs_c = quant_128x1_f32(dU, mode)
    dW1 = rows_scaled_gemm(dGq_c.T, dGs_c.T, xq_c.T, xs_c.T)
    dW3 = rows_scaled_gemm(dUq_c.T, dUs_c.T, xq_c.T, xs_c.T)
    dW13 = _f32(np.concatenate([dW1, dW3], axis=0))
    return dict(dx=dx, dW13=dW13, dW2=dW2, dh=dh, dG=dG, dU=dU, G=G, U=U, h=h, gh=gh)


def layer_backward(cf, x, Wr, bias, experts, dout, mode: int = SCALE_AMAX, details: bool = False) -> dict:
    """Backward of the layer's FFN part with the routing held fixed:
        out_t = u_t + FFN_shared(u_t) + sum_k g_{t,k} FFN_{e_{t,k}}(u_t)
    ("DeepSeek-V3 Technischer Bericht", Methode section 2, layer output
    equation).  Given dout [T, H] (bf16), each routed expert e receives, for
    every token t that selected it (slot k), dY = g_{t,k} * dout_t, handed to
    expert_backward as dout_t and the gate (the placement of g is described
    at the top of this module), the shared expert dY = dout; each runs
    expert_backward on its tokens in token order.
        dx_t = dout_t + dx_shared,t + sum_k dx_{e_{t,k}},t    (double, then FP32)
    The routing (and with it every gate) is the oracle's own; the gradient of
    the gates themselves (router backward) is not part of this.
    experts: list indexed by expert id (routed 0..N_r-1, shared N_r) of
    (W13q, s13, W2q, s2) tuples, None for experts no token uses.
    Returns dx [T, H], dW13 and dW2 dicts keyed by expert id (FP32 values as
    double arrays), and the routing (idx, gate, gap); with details, also
    per_expert: expert id -> (its tokens in order, expert_backward's dict)."""
    idx, gate, gap, _ = route(cf, x, Wr, bias)
    xu = _u16(x)
    d = _as_f32_values(dout)
    T = xu.shape[0]
    Nr = cf.Nr
    acc = d.astype(np.float64)
    dW13, dW2, per_expert = {}, {}, {}
    for e in range(Nr):
        toks, slots = np.nonzero(idx == e)
        if toks.size == 0:
            continue
        order = np.argsort(toks, kind="stable")
        toks, slots = toks[order], slots[order]
        r = expert_backward(xu[toks], d[toks], *experts[e], gate=gate[toks, slots], mode=mode)
        acc[toks] += r["dx"]
        dW13[e], dW2[e] = r["dW13"], r["dW2"]
        if details:
            per_expert[e] = (toks, r)
    if cf.Ns:
        r = expert_backward(xu, d, *experts[Nr], mode=mode)
        acc += r["dx"]
        dW13[Nr], dW2[Nr] = r["dW13"], r["dW2"]
        if details:
            per_expert[Nr] = (np.arange(T), r)
    out = dict(dx=_f32(acc), dW13=dW13, dW2=dW2, idx=idx, gate=gate, gap=gap)
    if details:
        out["per_expert"] = per_expert
    return out
