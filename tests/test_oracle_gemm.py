"""Pins of the oracle's block-scaled FP8 GEMM.

The pages ("DeepSeek-V3 Technischer Bericht", Kernideen FP8 bullet) fix
1x128 scales on activations, 128x128 scales on weights and FP32 promotion
every N_c = 128 accumulation steps: mathematically
C = sum_kb sA[m,kb] sB[n/128,kb] sum_{k in kb} A[m,k] B[n,k].  Pins: equality
with a dense double matmul of the dequantized operands (a library matmul), and
exactness of the per-block partial sums checked with integer arithmetic.
"""
import numpy as np

from moe_synth import gen_gemm_a, gen_gemm_b


def _operands(oracle_lib, M, K, N, seed):
    a = gen_gemm_a(M, K, seed)
    b = gen_gemm_b(K, N, seed).t().contiguous()  # [N, K]
    A, sA = oracle_lib.quant_1x128(a)
    B, sB = oracle_lib.quant_128x128(b)
    return A, sA, B, sB


def test_gemm_equals_dense_matmul_of_dequantized(oracle_lib):
    M, K, N = 48, 512, 256
    A, sA, B, sB = _operands(oracle_lib, M, K, N, 0)
    Cm = oracle_lib.blockscaled_gemm(A, sA, B, sB)
    Ad = oracle_lib.dequant(A, sA, 1)
    Bd = oracle_lib.dequant(B, sB, 128)
    ref = Ad @ Bd.T
    assert np.allclose(Cm, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_gemm_block_partials_exact(oracle_lib):
    # Unit scales: C * 2^18 must equal the exact integer product of the
    # codes' values on the 2^-9 grid.
    M, K, N = 16, 384, 128
    rng = np.random.default_rng(1)
    t = oracle_lib.e4m3_decode_table()
    finite = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    A = rng.choice(finite, size=(M, K)).astype(np.uint8)
    B = rng.choice(finite, size=(N, K)).astype(np.uint8)
    sA = np.ones((M, K // 128), np.float32)
    sB = np.ones((N // 128, K // 128), np.float32)
    Cm = oracle_lib.blockscaled_gemm(A, sA, B, sB)
    Ai = (t[A] * 512).astype(np.int64)
    Bi = (t[B] * 512).astype(np.int64)
    exact = Ai @ Bi.T
    assert np.array_equal(exact, exact)  # int64 headroom: |v| <= 448*512, K=384
    assert np.array_equal(np.round(Cm * 2.0 ** 18).astype(np.int64), exact)
    assert np.all(Cm * 2.0 ** 18 == exact.astype(np.float64))


def test_gemm_scale_indexing(oracle_lib):
    # Distinct scales per block: each must land on its own (row, kb) / (n/128, kb).
    M, K, N = 8, 256, 256
    rng = np.random.default_rng(2)
    A = np.full((M, K), 0x38, np.uint8)  # code 0x38 = 1.0
    B = np.full((N, K), 0x38, np.uint8)
    sA = rng.uniform(0.5, 2.0, (M, 2)).astype(np.float32)
    sB = rng.uniform(0.5, 2.0, (2, 2)).astype(np.float32)
    Cm = oracle_lib.blockscaled_gemm(A, sA, B, sB)
    for m in range(M):
        for n in range(N):
            want = 128.0 * (float(sA[m, 0]) * float(sB[n // 128, 0]) + float(sA[m, 1]) * float(sB[n // 128, 1]))
            assert Cm[m, n] == want
