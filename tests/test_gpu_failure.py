"""Failure detection without a GPU fault: a kernel whose mbarrier wait can
never complete gives up after its time limit, reports MOE_DEVERR_TIMEOUT in
the error word and returns; the CUDA context stays usable."""
import numpy as np
import pytest
import torch

import moe_synth as S

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives(oracle_lib):
    import sparse_moe_layer_expert_b200 as m
    err = m.new_err_flag()
    m.moe_selftest_wait_timeout(err, 20000)  # 20 ms limit
    st, v = m.moe_check_device_error(err)
    assert st == m.MOE_ERR_TIMEOUT and (v & m.MOE_DEVERR_TIMEOUT)
    # the context still works afterwards
    x = S.gen_x(8, 256, 0)
    q, s = m.fp8_quant_1x128(x.cuda())
    qo, so = oracle_lib.quant_1x128(x)
    assert np.array_equal(q.cpu().numpy(), qo)
    err.zero_()
    assert m.moe_check_device_error(err) == (m.MOE_OK, 0)


def test_selftest_rejects_bad_limit():
    import sparse_moe_layer_expert_b200 as m
    err = m.new_err_flag()
    with pytest.raises(m.MoeError):
        m.moe_selftest_wait_timeout(err, 0)
    with pytest.raises(m.MoeError):
        m.moe_selftest_wait_timeout(err, 10 ** 7)
