"""Shared helpers of the test suite: the comparison rule and problem builders.

Comparison rule (the layer's stated tolerance): floating outputs within a
relative Frobenius error of 2e-3 and a max |diff| of 1e-2 * rms(ref); for an
output stored as bf16, the format's own rounding (half a bf16 ulp of the
reference value) is added to the elementwise bound.  Integer and code
outputs compare bit-exactly.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import moe_synth as S

REL_FRO = 2e-3
MAX_REL_RMS = 1e-2
# Routing near-tie rule.  A token is exempt from the bit-exact comparison of
# its expert set when the oracle's gap between the last selected and the first
# rejected biased score is below NEAR_TIE.  The layer's stated rule uses 1e-5;
# on the V3-shaped workloads about 0.3% of tokens have such gaps (the top-8
# sigmoid scores crowd near 0.96, mean 8th/9th spacing ~3.6e-3), more than the
# 0.1% the rule tolerates, so the comparison uses the stricter 1e-6: every
# token with a gap of 1e-6 or more must match exactly and the exempt share
# stays well under 0.1%.  Tokens below the stated 1e-5 are still counted and
# reported.
NEAR_TIE = 1e-6
STATED_NEAR_TIE = 1e-5


def half_ulp_bf16(ref: np.ndarray) -> np.ndarray:
    a = np.abs(ref)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, np.exp2(e - 8), 2.0 ** -134)


def assert_close(got, ref, bf16_out: bool = False, what: str = "", rel_fro=REL_FRO, max_rel_rms=MAX_REL_RMS,
                 tie_allow=None):
    """The stated bound.  tie_allow (same shape as ref, or None): the largest
    change that E4M3 codes at a rounding near-tie of an FP32 intermediate
    (near_tie_steps) can make to each element, added to its max bound."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    d = got - ref
    nref = np.linalg.norm(ref)
    rms = math.sqrt(float(np.mean(ref * ref))) if ref.size else 0.0
    fro = np.linalg.norm(d) / nref if nref > 0 else np.linalg.norm(d)
    allow = max_rel_rms * rms + (half_ulp_bf16(ref) if bf16_out else 0.0)
    if tie_allow is not None:
        allow = allow + np.asarray(tie_allow, np.float64)
        n_tie = int((np.abs(d) > max_rel_rms * rms + (half_ulp_bf16(ref) if bf16_out else 0.0)).sum())
        if n_tie:
            print(f"{what}: {n_tie} elements beyond the stated max bound, within the near-tie allowance")
    bad = np.abs(d) > allow
    assert fro <= rel_fro, f"{what}: rel-Frobenius {fro:.3e} > {rel_fro}"
    assert not bad.any(), (f"{what}: {int(bad.sum())} elements beyond the bound; worst |d|="
                           f"{np.abs(d).max():.3e}, rms(ref)={rms:.3e}")
    return fro, float(np.abs(d).max()), rms


# Code near-ties of FP32 intermediates.  An intermediate that both sides
# compute in FP32 (h, dG, dU, g*h) carries a different rounding on each side,
# so where the oracle's quotient v/S lies within a small band of the midpoint
# between two E4M3 values, either code is a correct result, and the two differ
# by one code step.  Every element downstream of such a code may then differ
# by that step times the scale times the other GEMM operand's element: that
# much is added to its max bound (the relative Frobenius bound is unchanged).
# The band is the same as for the re-quantized h: relative to the midpoint
# above a quotient of 1, absolute below (the FP32 error of an accumulated
# value is of the size of its tile's scale, not of the value).
TIE_BAND = 1e-4
TIE_BAND_POW2 = 1e-3


def near_tie_steps(v: np.ndarray, S: np.ndarray, dec_table: np.ndarray, band: float = TIE_BAND) -> np.ndarray:
    """v: the oracle's FP32 values, S: the scale of each element's tile
    (broadcast to v's shape).  Returns, per element, 0 off a near-tie and
    |step| * S at one (the change in the dequantized value if the other side
    rounds to the other neighbour)."""
    v = np.asarray(v, np.float64)
    S = np.broadcast_to(np.asarray(S, np.float64), v.shape)
    grid = np.unique(np.abs(dec_table[np.isfinite(dec_table)]))
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.where(S > 0, np.abs(v) / np.where(S > 0, S, 1.0), 0.0)
    i = np.clip(np.searchsorted(grid, q, side="right"), 1, grid.size - 1)
    lo, hi = grid[i - 1], grid[i]
    mid = 0.5 * (lo + hi)
    near = (np.abs(q - mid) / np.maximum(mid, 1.0) <= band) & (S > 0)
    return np.where(near, (hi - lo) * S, 0.0)


def tiles_1x128(S_tiles: np.ndarray) -> np.ndarray:
    """[rows, C/128] scales -> per-element [rows, C]."""
    return np.repeat(np.asarray(S_tiles, np.float64), 128, axis=1)


def tiles_128x1(S_tiles: np.ndarray, rows: int) -> np.ndarray:
    """[ceil(rows/128), C] scales -> per-element [rows, C]."""
    return np.repeat(np.asarray(S_tiles, np.float64), 128, axis=0)[:rows]


def u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().float().numpy().astype(np.float64)


def shape_of(cfg: dict) -> dict:
    return {k: cfg[k] for k in ("H", "I", "Nr", "Kr", "Ns", "n_groups", "topk_groups", "scale_mode") if k in cfg}


def oracle_cfg(oracle, cfg: dict):
    return oracle.cfg(cfg["H"], cfg["I"], cfg["Nr"], cfg["Kr"], cfg.get("Ns", 1), cfg.get("n_groups", 0),
                      cfg.get("topk_groups", 0), cfg.get("route_scale", 1.0), cfg.get("scale_mode", 0))


def route_sets_match(idx_gpu: np.ndarray, idx_ref: np.ndarray, gap: np.ndarray):
    """Bit-exact routing up to near-ties: returns (mismatching tokens that are
    not exempt, number of exempt tokens)."""
    exempt = gap < NEAR_TIE
    bad = []
    for t in range(idx_ref.shape[0]):
        if exempt[t]:
            continue
        if set(idx_gpu[t].tolist()) != set(idx_ref[t].tolist()):
            bad.append(t)
    return bad, int(exempt.sum())


class Problem:
    """Seeded synthetic layer problem: bf16 inputs shared by the CUDA path
    and the oracle (which quantizes the weights itself)."""

    def __init__(self, cfg: dict, T: int, seed: int = 0, device="cpu", x_kind=None):
        self.cfg = dict(cfg)
        self.T = T
        self.seed = seed
        self.device = device
        H, Nr = cfg["H"], cfg["Nr"]
        kind = x_kind or cfg.get("x", "normal")
        if kind == "mixture":
            self.x, _ = S.gen_mixture_x(T, H, seed, device=device)
        else:
            self.x = S.gen_x(T, H, seed, device=device)
        self.wr = S.gen_router(Nr, H, seed, device=device)
        self.bias = S.gen_bias(Nr, seed, cfg.get("bias", "uniform"), device=device)
        self.E = Nr + cfg.get("Ns", 1)

    def expert_bf16(self, e: int):
        return S.gen_expert(e, self.cfg["H"], self.cfg["I"], self.seed, device=self.device)

    def oracle_expert(self, oracle, e: int):
        w13, w2 = self.expert_bf16(e)
        mode = self.cfg.get("scale_mode", 0)
        W13q, s13 = oracle.quant_128x128(w13, mode)
        W2q, s2 = oracle.quant_128x128(w2, mode)
        return W13q, s13, W2q, s2


GUARD = 4096        # guard band (bytes) around buffers the GPU tests hand to the library
GUARD_BYTE = 0xA5


def guarded_empty(shape, dtype, device="cuda"):
    """An uninitialised tensor inside a buffer with GUARD bytes of a fixed
    pattern on both sides; returns (tensor, check) where check() raises if a
    kernel wrote into either band."""
    esz = torch.empty((), dtype=dtype).element_size()
    n = 1
    for s in shape:
        n *= s
    nbytes = n * esz
    buf = torch.full((nbytes + 2 * GUARD,), GUARD_BYTE, dtype=torch.uint8, device=device)
    t = buf[GUARD:GUARD + nbytes].view(dtype).view(shape)

    def check():
        ok = bool((buf[:GUARD] == GUARD_BYTE).all()) and bool((buf[GUARD + nbytes:] == GUARD_BYTE).all())
        assert ok, f"guard band around a {tuple(shape)} {dtype} buffer overwritten"

    return t, check
