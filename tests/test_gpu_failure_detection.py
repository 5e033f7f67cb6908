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


@pytest.mark.parametrize("d,causal,B,H,N", [(64, False, 2, 4, 1000), (128, True, 2, 4, 1000),
                                           (64, True, 4, 40, 512)],
                         ids=["d64", "d128-causal", "d64-persistent"])
def test_forward_wait_limit_runs_out_and_context_survives(d, causal, B, H, N):
    # The forward kernel itself with a wait limit of a few cycles: some pipeline
    # wait runs out, every role of that CTA stops after its own copies and MMAs
    # have landed, and the call reports FA_ERR_DEVICE_TIMEOUT.  The context must
    # stay usable: a normal call afterwards passes parity and leaves the status clean.
    # The last case has 640 short blocks, so it runs the persistent CTA (the
    # scheduler, the mailbox and the block-to-block hand-offs wind down too).
    import torch
    from io_aware_exact_24_b200 import (FA_ERR_DEVICE_TIMEOUT, FA_OK, fa_get_device_status,
                                        fa_selftest_fwd_timeout)
    from fa_testutil import to_device_bf16
    assert fa_get_device_status() == FA_OK
    q = normal_bf16((B, H, N, d), 6 + d, 0)
    k = normal_bf16((B, H, N, d), 6 + d, 1)
    v = normal_bf16((B, H, N, d), 6 + d, 2)
    tq, tk, tv = to_device_bf16(q), to_device_bf16(k), to_device_bf16(v)
    o = torch.empty_like(tq)
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    scale = 1.0 / np.sqrt(d)
    for _ in range(2):
        st = fa_selftest_fwd_timeout(tq, tk, tv, o, lse, B, H, N, N, d, scale, causal, 2)
        assert st == FA_ERR_DEVICE_TIMEOUT
        assert fa_get_device_status() == FA_OK      # read and cleared by the call
    o2, lse2 = run_fa(q, k, v, scale, causal, None)
    o_ref, lse_ref = oracle.attn_ref(q, k, v, scale, causal, None)
    compare(o2, lse2, o_ref, lse_ref, f"after forward timeout d={d}")
    assert fa_get_device_status() == FA_OK


@pytest.mark.parametrize("d,causal,B,H,N", [(64, False, 1, 2, 700), (128, True, 1, 2, 700)],
                         ids=["d64", "d128-causal"])
def test_backward_wait_limit_runs_out_and_context_survives(d, causal, B, H, N):
    # The backward kernel with a wait limit of a few cycles: some pipeline wait runs
    # out, every role of that CTA stops after its own copies, MMAs and dQ reduce-adds
    # have landed, and the call reports FA_ERR_DEVICE_TIMEOUT.  Afterwards a normal
    # backward call passes its derived bound and leaves the status clean.  At d = 64
    # the kernel also copies K and V into TMEM, whose barrier winds down the same way.
    import torch
    from io_aware_exact_24_b200 import (FA_ERR_DEVICE_TIMEOUT, FA_OK, fa_bwd_workspace_size, fa_fwd,
                                        fa_get_device_status, fa_selftest_bwd_timeout)
    from fa_testutil import to_device_bf16
    from io_aware_exact_24_b200.inputs import TENSOR_DO
    from test_gpu_bwd import bounds, run_fwd_bwd
    assert fa_get_device_status() == FA_OK
    q = normal_bf16((B, H, N, d), 40 + d, 0)
    k = normal_bf16((B, H, N, d), 40 + d, 1)
    v = normal_bf16((B, H, N, d), 40 + d, 2)
    do = normal_bf16((B, H, N, d), 40 + d, TENSOR_DO)
    scale = float(np.float32(1 / np.sqrt(d)))
    tq, tk, tv, tdo = (to_device_bf16(x) for x in (q, k, v, do))
    o = torch.empty_like(tq)
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    fa_fwd(tq, tk, tv, o, lse, B, H, N, N, d, scale, causal, None)
    dq, dk, dv = torch.empty_like(tq), torch.empty_like(tk), torch.empty_like(tv)
    nbytes = fa_bwd_workspace_size(B, H, N, d)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    for _ in range(2):
        st = fa_selftest_bwd_timeout(tq, tk, tv, o, lse, tdo, dq, dk, dv, B, H, N, N, d, scale, causal,
                                     ws, nbytes, 2)
        assert st == FA_ERR_DEVICE_TIMEOUT
        assert fa_get_device_status() == FA_OK      # read and cleared by the call
    o2, lse2, gq, gk, gv = run_fwd_bwd(q, k, v, do, scale, causal, None)
    rq, rk, rv, bq, bk, bv, o_ref, lse_ref = bounds(q, k, v, do, scale, causal, None, o2, lse2)
    compare(o2, lse2, o_ref, lse_ref, f"forward after backward timeout d={d}")
    for name, g, r, bd in (("dQ", gq, rq, bq), ("dK", gk, rk, bk), ("dV", gv, rv, bv)):
        ratio = float((np.abs(g - r) / bd).max())
        assert ratio <= 1.0, f"after backward timeout d={d}: {name} at x{ratio:.3f} of its bound"
    assert fa_get_device_status() == FA_OK
