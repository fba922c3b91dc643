"""GPU parity of the 1x128 / 128x128 quantizers against the oracle: codes and
scales must be bit-identical ("DeepSeek-V3 Technischer Bericht", Kernideen FP8
bullet; "DeepSeek-V3 技術報告書", S = max|X|/448, clip(round(X/S)))."""
import numpy as np
import pytest
import torch

import moe_synth as S

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def m():
    import sparse_moe_layer_expert_b200 as pkg
    assert torch.cuda.is_available()
    return pkg


def _check_1x128(m, oracle_lib, x_cpu):
    q, s = m.fp8_quant_1x128(x_cpu.cuda())
    torch.cuda.synchronize()
    qo, so = oracle_lib.quant_1x128(x_cpu)
    qg = q.cpu().numpy()
    if not np.array_equal(qg, qo):
        r, c = np.nonzero(qg != qo)
        sg = s.cpu().numpy()
        xs = x_cpu.float().numpy()
        print("codes differ at", [(int(i), int(j), float(xs[i, j]), int(qg[i, j]), int(qo[i, j]),
                                   float(sg[i, j // 128]), float(so[i, j // 128])) for i, j in zip(r[:12], c[:12])])
    assert np.array_equal(qg, qo)
    assert np.array_equal(s.cpu().numpy(), so)


def test_1x128_ragged_outliers(m, oracle_lib):
    _check_1x128(m, oracle_lib, S.gen_gemm_a(333, 1024, 0))


def test_1x128_special_tiles(m, oracle_lib):
    x = S.gen_x(64, 512, 1)
    x[3, 128:256] = 0                      # all-zero tile -> S = 0, codes 0
    x[5, :128] = (x[5, :128].float() * 2.0 ** -30).to(torch.bfloat16)   # tiny magnitudes
    x[7, 256:384] = 3.0e4                  # constant tile
    x[9, 0] = -x[9, 0].abs() * 1000        # negative outlier
    x[11, 5] = -0.0
    # scales near and below the quantizer's switch from the reciprocal path to
    # the plain division (S < 2^-100): amax around 2^-91 .. 2^-125, bf16
    # subnormals included
    for i, e in enumerate((-91, -92, -100, -110, -120, -125, -130)):
        x[13 + i, 384:512] = (x[13 + i, 384:512].float() * 2.0 ** e).to(torch.bfloat16)
    _check_1x128(m, oracle_lib, x)


def test_1x128_strided_rows(m, oracle_lib):
    big = S.gen_x(40, 1024 + 64, 2)
    xv = big.cuda()[:, :1024]
    q, s = m.fp8_quant_1x128(xv)
    qo, so = oracle_lib.quant_1x128(big[:, :1024].contiguous())
    assert np.array_equal(q.cpu().numpy(), qo) and np.array_equal(s.cpu().numpy(), so)


def test_1x128_single_row(m, oracle_lib):
    _check_1x128(m, oracle_lib, S.gen_x(1, 128, 3))


def test_1x128_full_prefill_input(m, oracle_lib):
    _check_1x128(m, oracle_lib, S.gen_x(4096, 7168, 4))


def test_128x128_blocks(m, oracle_lib):
    w = S.normal_bf16((768, 1024), 0.02, 5)
    w[130, 7] = 1.5
    w[256:384, 128:256] = 0
    q, s = m.fp8_quant_128x128(w.cuda())
    qo, so = oracle_lib.quant_128x128(w)
    assert np.array_equal(q.cpu().numpy(), qo) and np.array_equal(s.cpu().numpy(), so)


def test_128x128_v3_expert(m, oracle_lib):
    w13, w2 = S.gen_expert(0, 7168, 2048, 6, device="cuda")
    for w in (w13, w2):
        q, s = m.fp8_quant_128x128(w)
        qo, so = oracle_lib.quant_128x128(w.cpu())
        assert np.array_equal(q.cpu().numpy(), qo) and np.array_equal(s.cpu().numpy(), so)


def test_quant_rejects_bad_arguments(m):
    x = torch.zeros((4, 200), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(m.MoeError) as e:
        m.fp8_quant_1x128(x)
    assert e.value.status == m.MOE_ERR_UNSUPPORTED_SHAPE
    x = torch.zeros((4, 129), dtype=torch.bfloat16, device="cuda")[:, 1:]
    with pytest.raises(m.MoeError) as e:  # misaligned base pointer
        m.fp8_quant_1x128(x.contiguous()[:, :] if False else x)
    assert e.value.status in (m.MOE_ERR_INVALID_ARG, m.MOE_ERR_UNSUPPORTED_SHAPE)


# ------------------------------------------------ power-of-two scale rule
def _check_1x128_pow2(m, oracle_lib, x_cpu):
    q, s = m.fp8_quant_1x128(x_cpu.cuda(), pow2=True)
    torch.cuda.synchronize()
    qo, so = oracle_lib.quant_1x128(x_cpu, 1)
    assert np.array_equal(s.cpu().numpy(), so)
    assert np.array_equal(q.cpu().numpy(), qo)


def test_1x128_pow2_ragged_outliers(m, oracle_lib):
    _check_1x128_pow2(m, oracle_lib, S.gen_gemm_a(333, 1024, 4))


def test_1x128_pow2_thresholds_and_special_tiles(m, oracle_lib):
    # tiles whose amax sits exactly on, just above and just below a threshold
    # 448 * 2^e, an all-zero tile, tiny (bf16-subnormal) and huge magnitudes
    x = S.gen_x(16, 1024, 5)
    for g, amax in enumerate([448.0, 450.0, 446.0, 224.0, 1.0, 2.0 ** -120, 3.0e38]):
        x[g, 128 * g:128 * g + 128] = (x[g, 128 * g:128 * g + 128].float().clamp(-0.5, 0.5) *
                                       (amax if amax < 1e30 else 1.0)).to(torch.bfloat16)
        x[g, 128 * g + 7] = amax
    x[9, 256:384] = 0
    x[10, :128] = (x[10, :128].float() * 2.0 ** -133).to(torch.bfloat16)
    _check_1x128_pow2(m, oracle_lib, x)


def test_128x128_pow2_blocks(m, oracle_lib):
    w = S.normal_bf16((384, 640), 0.02, 6)
    q, s = m.fp8_quant_128x128(w.cuda(), pow2=True)
    torch.cuda.synchronize()
    qo, so = oracle_lib.quant_128x128(w, 1)
    assert np.array_equal(s.cpu().numpy(), so)
    assert np.array_equal(q.cpu().numpy(), qo)
