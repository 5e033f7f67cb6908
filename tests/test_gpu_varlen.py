"""GPU parity of the packed variable-length forward (``fa_fwd_varlen``) against the
fp64 oracle evaluated sequence by sequence."""
import numpy as np
import pytest

import oracle
from io_aware_exact_24_b200.inputs import normal_bf16

from fa_testutil import compare, run_fa, to_device_bf16, to_host_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from io_aware_exact_24_b200.build import build
    build()


def run_varlen(q, k, v, cu_q, cu_k, scale, causal, max_q=None, guard=4096):
    import torch
    from io_aware_exact_24_b200 import fa_fwd_varlen
    Tq, H, d = q.shape
    Tk = k.shape[0]
    B = len(cu_q) - 1
    if max_q is None:
        max_q = int(np.diff(cu_q).max()) if B else 0
    tq, tk, tv = to_device_bf16(q), to_device_bf16(k), to_device_bf16(v)
    tcq = torch.from_numpy(np.asarray(cu_q, np.int32)).cuda()
    tck = torch.from_numpy(np.asarray(cu_k, np.int32)).cuda()
    n_o, n_l = Tq * H * d, Tq * H
    o_buf = torch.full((n_o + 2 * guard,), -12345.0, dtype=torch.bfloat16, device="cuda")
    l_buf = torch.full((n_l + 2 * guard,), -777.0, dtype=torch.float32, device="cuda")
    o = o_buf[guard:guard + n_o].view(Tq, H, d)
    lse = l_buf[guard:guard + n_l].view(Tq, H)
    fa_fwd_varlen(tq, tk if Tk else None, tv if Tk else None, o, lse, tcq, tck, B, H, Tq, Tk,
                  max_q, d, scale, causal)
    torch.cuda.synchronize()
    guards = bool((o_buf[:guard] == -12345.0).all() and (o_buf[guard + n_o:] == -12345.0).all()
                  and (l_buf[:guard] == -777.0).all() and (l_buf[guard + n_l:] == -777.0).all())
    return to_host_f64(o), lse.cpu().numpy().astype(np.float64), guards


CASES = [
    # H, d, causal, query lengths, key lengths (None: same as the query lengths)
    (2, 64, True, [1, 127, 128, 129, 300], None),
    (3, 128, True, [513, 0, 64, 1000], None),
    (2, 128, False, [200, 5, 381], [17, 700, 381]),
    (4, 64, True, [100, 260], [300, 90]),        # N_q < N_k and N_q > N_k per sequence
    (1, 128, False, [0, 0, 77], [0, 12, 0]),     # empty sequences, a sequence without keys
]


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_varlen_matches_oracle(case):
    H, d, causal, lq, lk = case
    lk = lq if lk is None else lk
    cu_q = np.concatenate([[0], np.cumsum(lq)]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum(lk)]).astype(np.int32)
    Tq, Tk = int(cu_q[-1]), int(cu_k[-1])
    seed = 900 + Tq + Tk + d
    q = normal_bf16((Tq, H, d), seed, 0)
    k = normal_bf16((Tk, H, d), seed, 1)
    v = normal_bf16((Tk, H, d), seed, 2)
    scale = 1.0 / np.sqrt(d)
    o, lse, guards = run_varlen(q, k, v, cu_q, cu_k, scale, causal)
    assert guards, "wrote outside O / LSE"
    o_ref, lse_ref = oracle.attn_ref_varlen(q, k, v, cu_q, cu_k, scale, causal)
    errs = compare(o, lse, o_ref, lse_ref, str(case))
    print(f"{case}: max|dO|={errs[0]:.3e} relF={errs[1]:.3e} max|dLSE|={errs[2]:.3e}")


def test_equal_lengths_are_bitwise_the_dense_forward():
    B, H, N, d = 3, 2, 300, 128
    q = normal_bf16((B, H, N, d), 84, 0)
    k = normal_bf16((B, H, N, d), 84, 1)
    v = normal_bf16((B, H, N, d), 84, 2)
    a = {}
    run_fa(q, k, v, 0.09, True, None, out=a)
    pack = lambda x: np.ascontiguousarray(x.transpose(0, 2, 1, 3).reshape(B * N, H, d))
    cu = (np.arange(B + 1) * N).astype(np.int32)
    o, lse, _ = run_varlen(pack(q), pack(k), pack(v), cu, cu, 0.09, True)
    from io_aware_exact_24_b200.inputs import bf16_bits_to_f32
    dense = bf16_bits_to_f32(a["o_bits"].view(np.uint16)).astype(np.float64)
    assert np.array_equal(o, dense.transpose(0, 2, 1, 3).reshape(B * N, H, d))
    assert np.array_equal(lse.astype(np.float32).view(np.uint32),
                          np.ascontiguousarray(a["lse_raw"].transpose(0, 2, 1).reshape(B * N, H)).view(np.uint32))
