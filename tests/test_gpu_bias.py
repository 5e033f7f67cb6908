"""GPU parity of the additive-positional-bias forward (``fa_fwd_bias``) against the
fp64 oracle's biased definition."""
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


def alibi_slopes(H):
    """The usual geometric per-head slopes 2^(-8(h+1)/H)."""
    return (2.0 ** (-8.0 * (np.arange(H) + 1) / H)).astype(np.float32)


def run_bias(q, k, v, scale, causal, key_lens, slopes, W=-1, out=None):
    import torch
    from io_aware_exact_24_b200 import fa_fwd_bias
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    tq, tk, tv = to_device_bf16(q), to_device_bf16(k), to_device_bf16(v)
    tkl = None if key_lens is None else torch.from_numpy(np.asarray(key_lens, np.int32)).cuda()
    ts = torch.from_numpy(np.asarray(slopes, np.float32)).cuda()
    o = torch.empty((B, H, Nq, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device="cuda")
    fa_fwd_bias(tq, tk if Nk else None, tv if Nk else None, o, lse, B, H, Nq, Nk, d, scale, causal,
                tkl, ts, W)
    torch.cuda.synchronize()
    if out is not None:
        out["o_bits"] = o.view(torch.int16).cpu().numpy()
        out["lse_raw"] = lse.cpu().numpy()
    return to_host_f64(o), lse.cpu().numpy().astype(np.float64)


CASES = [
    # B, H, Nq, Nk, d, causal, key_lens, W
    (1, 4, 1000, 1000, 128, True, None, -1),
    (2, 8, 700, 700, 64, True, None, -1),
    (2, 4, 300, 900, 64, False, [900, 400], -1),     # non-causal: |distance| both sides
    (1, 2, 1100, 1100, 128, True, None, 256),        # with a sliding window
    (1, 2, 400, 150, 64, True, None, -1),            # leading rows see nothing
]


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_bias_matches_oracle(case):
    B, H, Nq, Nk, d, causal, kl, W = case
    seed = 800 + Nq + Nk + d
    q = normal_bf16((B, H, Nq, d), seed, 0)
    k = normal_bf16((B, H, Nk, d), seed, 1)
    v = normal_bf16((B, H, Nk, d), seed, 2)
    kl_arr = None if kl is None else np.array(kl, np.int32)
    slopes = alibi_slopes(H)
    scale = 1.0 / np.sqrt(d)
    o, lse = run_bias(q, k, v, scale, causal, kl_arr, slopes, W)
    o_ref, lse_ref = oracle.attn_ref_bias(q, k, v, scale, slopes, causal, kl_arr, W)
    errs = compare(o, lse, o_ref, lse_ref, str(case))
    print(f"{case}: max|dO|={errs[0]:.3e} relF={errs[1]:.3e} max|dLSE|={errs[2]:.3e}")


def test_zero_slopes_agree_with_the_plain_forward():
    B, H, Nq, Nk, d = 2, 2, 333, 700, 128
    q = normal_bf16((B, H, Nq, d), 83, 0)
    k = normal_bf16((B, H, Nk, d), 83, 1)
    v = normal_bf16((B, H, Nk, d), 83, 2)
    o_a, l_a = run_fa(q, k, v, 0.09, True, None)
    o_b, l_b = run_bias(q, k, v, 0.09, True, None, np.zeros(H, np.float32))
    # the biased path forms s*c before the max instead of inside the exponent's
    # fused multiply-add, so P can round differently in its last bf16 bit
    assert np.abs(o_a - o_b).max() <= 4e-3
    assert np.abs(l_a - l_b).max() <= 1e-5


# ---------------------------------------------------------------- custom positional bias table

def run_table(q, k, v, scale, causal, key_lens, table, W=-1, guard=4096):
    import torch
    from io_aware_exact_24_b200 import fa_fwd_bias_table
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    tq, tk, tv = to_device_bf16(q), to_device_bf16(k), to_device_bf16(v)
    tkl = None if key_lens is None else torch.from_numpy(np.asarray(key_lens, np.int32)).cuda()
    tab = np.ascontiguousarray(table, np.float32)
    R = (tab.shape[1] - 1) // 2
    # the table sits between guard values that would show up in O if read
    tbuf = torch.full((tab.size + 2 * guard,), 1e4, dtype=torch.float32, device="cuda")
    tbuf[guard:guard + tab.size] = torch.from_numpy(tab.reshape(-1)).cuda()
    tt = tbuf[guard:guard + tab.size]
    o = torch.empty((B, H, Nq, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device="cuda")
    fa_fwd_bias_table(tq, tk if Nk else None, tv if Nk else None, o, lse, B, H, Nq, Nk, d, scale,
                      causal, tkl, tt, R, W)
    torch.cuda.synchronize()
    return to_host_f64(o), lse.cpu().numpy().astype(np.float64)


def _table(H, R, seed, sigma=1.0):
    return (np.random.default_rng(seed).standard_normal((H, 2 * R + 1)) * sigma).astype(np.float32)


TABLE_CASES = [
    # B, H, Nq, Nk, d, causal, key_lens, W, R
    (1, 4, 1000, 1000, 128, True, None, -1, 1000),     # every relative position in the table
    (2, 3, 700, 700, 64, True, None, -1, 96),          # clamped beyond +-96
    (2, 2, 300, 900, 64, False, [900, 400], -1, 128),  # non-causal, both signs, padded keys
    (1, 2, 1100, 1100, 128, True, None, 256, 300),     # with a sliding window
    (1, 2, 400, 150, 64, True, None, -1, 0),           # R = 0: one constant per head
    (2, 2, 129, 257, 128, False, None, -1, 5),         # ragged tiles, tight clamp
]


@pytest.mark.parametrize("case", TABLE_CASES, ids=[str(c) for c in TABLE_CASES])
def test_bias_table_matches_oracle(case):
    B, H, Nq, Nk, d, causal, kl, W, R = case
    seed = 850 + Nq + Nk + d + R
    q = normal_bf16((B, H, Nq, d), seed, 0)
    k = normal_bf16((B, H, Nk, d), seed, 1)
    v = normal_bf16((B, H, Nk, d), seed, 2)
    kl_arr = None if kl is None else np.array(kl, np.int32)
    table = _table(H, R, seed)
    scale = 1.0 / np.sqrt(d)
    o, lse = run_table(q, k, v, scale, causal, kl_arr, table, W)
    o_ref, lse_ref = oracle.attn_ref_bias_table(q, k, v, scale, table, causal, kl_arr, W)
    errs = compare(o, lse, o_ref, lse_ref, str(case))
    print(f"{case}: max|dO|={errs[0]:.3e} relF={errs[1]:.3e} max|dLSE|={errs[2]:.3e}")


def test_linear_table_is_the_slope_bias():
    # a table holding -m*|r| with R beyond every distance is the slope bias
    B, H, N, d = 1, 4, 900, 64
    q = normal_bf16((B, H, N, d), 861, 0)
    k = normal_bf16((B, H, N, d), 861, 1)
    v = normal_bf16((B, H, N, d), 861, 2)
    slopes = alibi_slopes(H)
    R = N
    r = np.arange(-R, R + 1, dtype=np.float64)
    table = (-slopes[:, None].astype(np.float64) * np.abs(r)[None, :]).astype(np.float32)
    o_t, l_t = run_table(q, k, v, 0.125, True, None, table)
    o_s, l_s = run_bias(q, k, v, 0.125, True, None, slopes)
    assert np.abs(o_t - o_s).max() <= 4e-3
    assert np.abs(l_t - l_s).max() <= 1e-4
