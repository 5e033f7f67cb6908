"""Failure detection on the GPU without a fault: a bounded wait on a barrier
nothing arrives on must give up, report FA_ERR_DEVICE_TIMEOUT through the
host status call, and leave the context usable."""
import numpy as np
import pytest

import oracle
from io_aware_exact_24_b200.inputs import normal_bf16

from fa_testutil import compare, run_fa

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def test_bounded_wait_reports_timeout_and_context_survives():
    from io_aware_exact_24_b200 import (FA_ERR_DEVICE_TIMEOUT, FA_OK, fa_get_device_status,
                                        fa_selftest_wait_timeout)
    assert fa_get_device_status() == FA_OK
    assert fa_selftest_wait_timeout(1 << 20) == FA_ERR_DEVICE_TIMEOUT
    assert fa_get_device_status() == FA_OK          # the status word was cleared
    q = normal_bf16((1, 2, 130, 64), 5, 0)
    k = normal_bf16((1, 2, 130, 64), 5, 1)
    v = normal_bf16((1, 2, 130, 64), 5, 2)
    o, lse = run_fa(q, k, v, 0.125, True, None)
    o_ref, lse_ref = oracle.attn_ref(q, k, v, 0.125, True, None)
    compare(o, lse, o_ref, lse_ref, "after timeout")
    assert fa_get_device_status() == FA_OK
