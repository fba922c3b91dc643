"""Seeded synthetic inputs for the FP8 DeepSeekMoE layer.

This module draws random tensors and nothing else: it holds none of the
layer's arithmetic (no quantization, routing, GEMM or combine), so both the
CUDA path and the CPU oracle can take their inputs from it.  Shapes and value
distributions follow the model the DeepSeek-V3 pages describe (hidden 7168,
expert intermediate 2048, 256 routed + 1 shared experts, top-8) and the small
configurations used for parity.

Every generator takes an explicit seed and device; the same (seed, device)
gives the same bytes.  Per-expert weights get their own seed so any single
expert can be regenerated without drawing the others.
"""
from __future__ import annotations

import math

import torch

# Layer shapes.  T tokens, H hidden, I expert intermediate, Nr routed experts,
# Kr experts per token, Ns shared experts, optional group-limited routing.
TINY = dict(name="tiny", T=256, H=512, I=256, Nr=16, Kr=4, Ns=1, n_groups=0, topk_groups=0,
            bias="uniform", x="normal")
_V3 = dict(H=7168, I=2048, Nr=256, Kr=8, Ns=1, n_groups=0, topk_groups=0)
DECODE = dict(_V3, name="decode", T=64, bias="zero", x="normal")
PREFILL = dict(_V3, name="prefill", T=4096, bias="uniform", x="normal")
SKEWED = dict(_V3, name="skewed", T=16384, n_groups=8, topk_groups=4, bias="zero", x="mixture")
# Standalone block-scaled GEMM shapes (M, K, N).
GEMM_SHAPES = [(4096, 7168, 4096), (4096, 2048, 7168)]

CONFIGS = {c["name"]: c for c in (TINY, DECODE, PREFILL, SKEWED)}

WEIGHT_STD = 0.02
BIAS_RANGE = 0.01


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) & 0x7FFFFFFFFFFFFFFF)
    return g


def _sub_seed(seed: int, *salt: int) -> int:
    h = int(seed) * 1000003
    for s in salt:
        h = (h ^ (int(s) + 0x9E3779B9)) * 1000003 & 0x7FFFFFFFFFFFFFFF
    return h


def normal_bf16(shape, std: float, seed: int, device="cpu") -> torch.Tensor:
    g = _gen(seed, device)
    return (torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std).to(torch.bfloat16)


def gen_x(T: int, H: int, seed: int, device="cpu") -> torch.Tensor:
    """Hidden states u_t ~ N(0, 1), bf16 [T, H]."""
    return normal_bf16((T, H), 1.0, _sub_seed(seed, 1), device)


def gen_mixture_x(T: int, H: int, seed: int, device="cpu", n_centroids: int = 32, zipf_s: float = 1.0,
                  noise: float = 0.3) -> tuple[torch.Tensor, torch.Tensor]:
    """Hidden states from a Gaussian mixture with Zipf-distributed component
    weights: x = c_z + noise * N(0, I), c ~ N(0, I), P(z = k) ~ 1/(k+1)^s.
    Returns (x bf16 [T, H], z int64 [T])."""
    g = _gen(_sub_seed(seed, 2), device)
    cent = torch.randn((n_centroids, H), generator=g, device=device)
    w = torch.tensor([1.0 / math.pow(k + 1, zipf_s) for k in range(n_centroids)], device=device)
    z = torch.multinomial(w / w.sum(), T, replacement=True, generator=g)
    x = cent[z] + noise * torch.randn((T, H), generator=g, device=device)
    return x.to(torch.bfloat16), z


def gen_router(Nr: int, H: int, seed: int, device="cpu") -> torch.Tensor:
    """Router centroids e_i ~ N(0, 0.02^2), bf16 [Nr, H]."""
    return normal_bf16((Nr, H), WEIGHT_STD, _sub_seed(seed, 3), device)


def gen_bias(Nr: int, seed: int, kind: str = "uniform", device="cpu") -> torch.Tensor:
    """Selection bias b_i, f32 [Nr]: zeros or U(-0.01, 0.01)."""
    if kind == "zero":
        return torch.zeros(Nr, dtype=torch.float32, device=device)
    g = _gen(_sub_seed(seed, 4), device)
    return (torch.rand(Nr, generator=g, device=device) * 2.0 - 1.0) * BIAS_RANGE


def gen_expert(e: int, H: int, I: int, seed: int, device="cpu") -> tuple[torch.Tensor, torch.Tensor]:
    """Expert e's bf16 weights, each entry ~ N(0, 0.02^2):
    W13 [2I, H] (rows 0..I-1 gate projection W1, rows I..2I-1 up projection
    W3) and W2 [H, I] (down projection).  Experts 0..Nr-1 are routed, Nr.. are
    shared."""
    w13 = normal_bf16((2 * I, H), WEIGHT_STD, _sub_seed(seed, 5, e), device)
    w2 = normal_bf16((H, I), WEIGHT_STD, _sub_seed(seed, 6, e), device)
    return w13, w2


def gen_gemm_a(M: int, K: int, seed: int, device="cpu", outlier_p: float = 0.01,
               outlier_mult: float = 50.0) -> torch.Tensor:
    """GEMM activations ~ N(0, 1) with a Bernoulli(1%) subset multiplied by 50,
    bf16 [M, K]."""
    g = _gen(_sub_seed(seed, 7), device)
    a = torch.randn((M, K), generator=g, device=device)
    mask = torch.rand((M, K), generator=g, device=device) < outlier_p
    a = torch.where(mask, a * outlier_mult, a)
    return a.to(torch.bfloat16)


def gen_gemm_b(K: int, N: int, seed: int, device="cpu") -> torch.Tensor:
    """GEMM weights B [K, N] ~ N(0, 0.02^2), bf16."""
    return normal_bf16((K, N), WEIGHT_STD, _sub_seed(seed, 8), device)
