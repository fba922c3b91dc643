"""GPU parity of the standalone block-scaled FP8 GEMM (tcgen05) against the
oracle's double-precision block-scaled product ("DeepSeek-V3 Technischer
Bericht", Kernideen: 1x128 activation scales, 128x128 weight scales, FP32
promotion every 128 K).  The output is bf16, so the comparison allows the
format's own rounding on top of the stated tolerance."""
import numpy as np
import pytest
import torch

import moe_synth as S
from _moe_util import assert_close, bf16_to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def m():
    import sparse_moe_layer_expert_b200 as pkg
    return pkg


def _operands(m, oracle_lib, M, K, N, seed):
    a = S.gen_gemm_a(M, K, seed, device="cuda")
    b = S.gen_gemm_b(K, N, seed, device="cuda").t().contiguous()
    A, sA = m.fp8_quant_1x128(a)
    B, sB = m.fp8_quant_128x128(b)
    return a, b, A, sA, B, sB


@pytest.mark.parametrize("M,N,K", [(1, 128, 128), (16, 256, 256), (37, 384, 256), (300, 512, 1024),
                                   (129, 256, 7168), (256, 1152, 2048)])
def test_gemm_matches_oracle(m, oracle_lib, M, N, K):
    a, b, A, sA, B, sB = _operands(m, oracle_lib, M, K, N, M * 7 + N)
    err = m.new_err_flag()
    C = m.fp8_blockscaled_gemm(A, sA, B, sB, err=err)
    assert m.moe_check_device_error(err)[0] == m.MOE_OK
    ref = oracle_lib.blockscaled_gemm(A.cpu().numpy(), sA.cpu().numpy(), B.cpu().numpy(), sB.cpu().numpy())
    assert_close(bf16_to_f64(C), ref, bf16_out=True, what=f"gemm {M}x{N}x{K}")


@pytest.mark.parametrize("M,K,N", S.GEMM_SHAPES)
def test_gemm_full_size_sampled_rows(m, oracle_lib, M, K, N):
    a, b, A, sA, B, sB = _operands(m, oracle_lib, M, K, N, 11)
    err = m.new_err_flag()
    C = m.fp8_blockscaled_gemm(A, sA, B, sB, err=err)
    assert m.moe_check_device_error(err)[0] == m.MOE_OK
    rows = np.sort(np.random.default_rng(0).choice(M, 48, replace=False))
    rows = np.unique(np.concatenate([rows, [0, 127, 128, M - 1]]))
    Ah, sAh = A.cpu().numpy()[rows], sA.cpu().numpy()[rows]
    ref = oracle_lib.blockscaled_gemm(Ah, sAh, B.cpu().numpy(), sB.cpu().numpy())
    assert_close(bf16_to_f64(C[torch.as_tensor(rows, device="cuda")]), ref, bf16_out=True, what="gemm full")
    # the quantized operands themselves are the oracle's, bit for bit
    qo, so = oracle_lib.quant_1x128(a[torch.as_tensor(rows, device="cuda")].cpu())
    assert np.array_equal(Ah, qo) and np.array_equal(sAh, so)


def test_gemm_rejects_bad_shapes(m):
    A = torch.zeros((4, 200), dtype=torch.uint8, device="cuda")
    sA = torch.zeros((4, 2), device="cuda")
    B = torch.zeros((128, 200), dtype=torch.uint8, device="cuda")
    with pytest.raises(m.MoeError) as e:
        m.fp8_blockscaled_gemm(A, sA, B, sA)
    assert e.value.status == m.MOE_ERR_UNSUPPORTED_SHAPE
