"""GPU parity of the sliding-window forward (``fa_fwd_window``) against the fp64
oracle's windowed definition."""
import numpy as np
import pytest

import oracle
from io_aware_exact_24_b200.inputs import bf16_bits_to_f32, normal_bf16

from fa_testutil import compare, run_fa, to_device_bf16, to_host_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from io_aware_exact_24_b200.build import build
    build()


def run_window(q, k, v, scale, causal, key_lens, W, out=None):
    import torch
    from io_aware_exact_24_b200 import fa_fwd_window
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    tq, tk, tv = to_device_bf16(q), to_device_bf16(k), to_device_bf16(v)
    tkl = None if key_lens is None else torch.from_numpy(np.asarray(key_lens, np.int32)).cuda()
    g = 2048
    o_buf = torch.full((B * H * Nq * d + 2 * g,), -12345.0, dtype=torch.bfloat16, device="cuda")
    l_buf = torch.full((B * H * Nq + 2 * g,), -777.0, dtype=torch.float32, device="cuda")
    o = o_buf[g:g + B * H * Nq * d].view(B, H, Nq, d)
    lse = l_buf[g:g + B * H * Nq].view(B, H, Nq)
    fa_fwd_window(tq, tk if Nk else None, tv if Nk else None, o, lse, B, H, Nq, Nk, d, scale,
                  causal, tkl, W)
    torch.cuda.synchronize()
    assert bool((o_buf[:g] == -12345.0).all() and (o_buf[g + o.numel():] == -12345.0).all())
    assert bool((l_buf[:g] == -777.0).all() and (l_buf[g + lse.numel():] == -777.0).all())
    if out is not None:
        out["o_bits"] = o.view(torch.int16).cpu().numpy()
        out["lse_raw"] = lse.cpu().numpy()
    return to_host_f64(o), lse.cpu().numpy().astype(np.float64)


CASES = [
    # B, H, Nq, Nk, d, causal, key_lens, W
    (1, 2, 1000, 1000, 128, True, None, 256),
    (2, 2, 700, 700, 64, True, None, 100),       # window inside one tile, crossing tiles
    (1, 1, 1100, 1100, 64, True, None, 127),
    (1, 1, 1100, 1100, 128, True, None, 128),
    (2, 1, 513, 2000, 64, True, [2000, 900], 300),   # N_q < N_k, key_lens cut some windows
    (1, 2, 400, 150, 128, True, None, 40),       # N_q > N_k: leading rows see nothing
    (2, 2, 300, 800, 64, False, None, 200),      # non-causal: lower bound only
    (1, 3, 260, 260, 128, True, None, 0),        # diagonal only
    (1, 1, 64, 0, 64, True, None, 5),            # no keys
]


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_window_matches_oracle(case):
    B, H, Nq, Nk, d, causal, kl, W = case
    seed = 700 + Nq + Nk + d + W
    q = normal_bf16((B, H, Nq, d), seed, 0)
    k = normal_bf16((B, H, Nk, d), seed, 1)
    v = normal_bf16((B, H, Nk, d), seed, 2)
    kl_arr = None if kl is None else np.array(kl, np.int32)
    scale = 1.0 / np.sqrt(d)
    o, lse = run_window(q, k, v, scale, causal, kl_arr, W)
    o_ref, lse_ref = oracle.attn_ref_window(q, k, v, scale, W, causal, kl_arr)
    errs = compare(o, lse, o_ref, lse_ref, str(case))
    print(f"{case}: max|dO|={errs[0]:.3e} relF={errs[1]:.3e} max|dLSE|={errs[2]:.3e}")


def test_window_zero_returns_the_diagonal_value_rows():
    B, H, N, d = 2, 2, 300, 64
    q = normal_bf16((B, H, N, d), 81, 0)
    k = normal_bf16((B, H, N, d), 81, 1)
    v = normal_bf16((B, H, N, d), 81, 2)
    o, _ = run_window(q, k, v, 0.125, True, None, 0)
    assert np.array_equal(o, bf16_bits_to_f32(v).astype(np.float64))


def test_wide_window_is_bitwise_the_plain_forward():
    B, H, Nq, Nk, d = 2, 2, 333, 700, 128
    q = normal_bf16((B, H, Nq, d), 82, 0)
    k = normal_bf16((B, H, Nk, d), 82, 1)
    v = normal_bf16((B, H, Nk, d), 82, 2)
    a, b = {}, {}
    run_fa(q, k, v, 0.09, True, None, out=a)
    run_window(q, k, v, 0.09, True, None, Nk, out=b)
    assert np.array_equal(a["o_bits"], b["o_bits"])
    assert np.array_equal(a["lse_raw"].view(np.uint32), b["lse_raw"].view(np.uint32))
