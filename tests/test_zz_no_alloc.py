"""GPU test of fa_fwd_splitkv_noalloc, the split-KV entry point that allocates
nothing (its workspace is the library's own file-scope device scratch).

Collected last on purpose.  Two calls in a row must each give, bit for bit, what
fa_fwd_splitkv gives with a caller-provided workspace on the same inputs; a
problem whose workspace exceeds the scratch is rejected before any launch.
"""
import numpy as np
import pytest

from io_aware_exact_24_b200.inputs import normal_bf16

from fa_testutil import to_device_bf16

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 16 << 20


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from io_aware_exact_24_b200.build import build
    build()


def _problem(B, H, Nq, Nk, d, seed):
    return (to_device_bf16(normal_bf16((B, H, Nq, d), seed, 0)),
            to_device_bf16(normal_bf16((B, H, Nk, d), seed, 1)),
            to_device_bf16(normal_bf16((B, H, Nk, d), seed, 2)))


def _with_workspace(q, k, v, scale, causal, kl, S):
    import torch
    from io_aware_exact_24_b200 import fa_fwd_splitkv, fa_fwd_splitkv_workspace_size
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device="cuda")
    n = fa_fwd_splitkv_workspace_size(B, H, Nq, d, S)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    fa_fwd_splitkv(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal, kl, S, ws, n)
    return o, lse


def _no_alloc(q, k, v, scale, causal, kl, S):
    import torch
    from io_aware_exact_24_b200 import fa_fwd_splitkv_noalloc
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device="cuda")
    fa_fwd_splitkv_noalloc(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal, kl, S)
    return o, lse


def test_two_calls_in_a_row_match_the_workspace_entry_point():
    import torch
    # two different problems back to back on one stream: the second call reuses
    # the scratch the first one wrote
    first = (_problem(2, 4, 3, 3000, 128, 900), 0.088, True, None, 7)
    kl = torch.tensor([700, 1], dtype=torch.int32, device="cuda")
    second = (_problem(2, 3, 1, 5000, 64, 901), 0.125, False, kl, 12)
    outs = []
    for (q, k, v), scale, causal, klen, S in (first, second):
        outs.append(_no_alloc(q, k, v, scale, causal, klen, S))
    torch.cuda.synchronize()
    for ((q, k, v), scale, causal, klen, S), (o_na, l_na) in zip((first, second), outs):
        o_ws, l_ws = _with_workspace(q, k, v, scale, causal, klen, S)
        torch.cuda.synchronize()
        assert torch.equal(o_na.view(torch.int16), o_ws.view(torch.int16))
        assert np.array_equal(l_na.cpu().numpy().view(np.uint32), l_ws.cpu().numpy().view(np.uint32))


def test_oversize_problem_is_rejected_before_launch():
    from io_aware_exact_24_b200 import FA_ERR_UNSUPPORTED, fa_fwd_splitkv_noalloc
    from io_aware_exact_24_b200 import fa_fwd_splitkv_workspace_size
    B, H, Nq, d, S = 8, 32, 128, 128, 2   # 2*8*32*128 rows x (128+1) floats > 16 MiB
    assert fa_fwd_splitkv_workspace_size(B, H, Nq, d, S) > SCRATCH_BYTES
    P = 1 << 20   # never dereferenced: the size check comes first
    st = fa_fwd_splitkv_noalloc(P, P, P, P, P, B, H, Nq, 64, d, 0.1, False, None, S, check=False)
    assert st == FA_ERR_UNSUPPORTED
