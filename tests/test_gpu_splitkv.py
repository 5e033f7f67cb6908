"""GPU parity of the split-KV forward (``fa_fwd_splitkv``) against the fp64 oracle.

Decode-shaped problems (a few query rows, long keys), ranges that are empty,
more ranges than K/V tiles, masks that empty whole rows, and agreement with the
single-pass forward on the same inputs.
"""
import numpy as np
import pytest

import oracle
from io_aware_exact_24_b200.inputs import DECODE_WORKLOADS, make_inputs, normal_bf16

from fa_testutil import compare, run_fa, to_device_bf16, to_host_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from io_aware_exact_24_b200.build import build
    build()


def run_splitkv(q, k, v, scale, causal, key_lens, num_splits, guard=4096):
    """fa_fwd_splitkv on bf16 bit arrays; returns (O f64, LSE f64, guards intact)."""
    import torch
    from io_aware_exact_24_b200 import (fa_fwd_splitkv, fa_fwd_splitkv_workspace_size,
                                        fa_splitkv_num_splits)
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    if num_splits == "auto":
        num_splits = fa_splitkv_num_splits(B, H, Nq, Nk)
    tq, tk, tv = to_device_bf16(q), to_device_bf16(k), to_device_bf16(v)
    tkl = None if key_lens is None else torch.from_numpy(np.asarray(key_lens, np.int32)).cuda()
    n_o, n_l = B * H * Nq * d, B * H * Nq
    o_buf = torch.full((n_o + 2 * guard,), -12345.0, dtype=torch.bfloat16, device="cuda")
    l_buf = torch.full((n_l + 2 * guard,), -777.0, dtype=torch.float32, device="cuda")
    o = o_buf[guard:guard + n_o].view(B, H, Nq, d)
    lse = l_buf[guard:guard + n_l].view(B, H, Nq)
    ws_bytes = fa_fwd_splitkv_workspace_size(B, H, Nq, d, num_splits)
    # garbage in the workspace must not matter: every partial is written before it is read
    ws = torch.full((ws_bytes // 4 + 64,), float("nan"), dtype=torch.float32, device="cuda")
    fa_fwd_splitkv(tq, tk if Nk else None, tv if Nk else None, o, lse, B, H, Nq, Nk, d, scale,
                   causal, tkl, num_splits, ws, ws_bytes)
    torch.cuda.synchronize()
    guards = bool((o_buf[:guard] == -12345.0).all() and (o_buf[guard + n_o:] == -12345.0).all()
                  and (l_buf[:guard] == -777.0).all() and (l_buf[guard + n_l:] == -777.0).all())
    return to_host_f64(o), lse.cpu().numpy().astype(np.float64), guards


CASES = [
    # B, H, Nq, Nk, d, causal, key_lens, num_splits
    (2, 4, 1, 4097, 128, False, None, 8),
    (1, 8, 1, 16384, 64, False, None, "auto"),
    (3, 2, 5, 1000, 64, True, None, 3),
    (2, 2, 16, 3000, 128, True, [1500, 3000], 7),
    (1, 1, 1, 1, 64, False, None, 4),            # more ranges than K/V tiles
    (1, 3, 2, 130, 128, False, None, 16),        # two tiles, sixteen ranges
    (2, 1, 200, 600, 128, False, None, 2),       # two query blocks
    (1, 2, 3, 0, 64, False, None, 2),            # no keys at all
    (2, 2, 1, 700, 64, False, [0, 5], 3),        # batch 0 sees no key
    (1, 1, 300, 100, 128, True, None, 3),        # N_q > N_k causal: leading rows see no key
    (4, 2, 7, 2049, 64, True, [2049, 1, 128, 129], 5),
]


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_splitkv_matches_oracle(case):
    B, H, Nq, Nk, d, causal, kl, S = case
    seed = 500 + Nq + Nk + d
    q = normal_bf16((B, H, Nq, d), seed, 0)
    k = normal_bf16((B, H, Nk, d), seed, 1)
    v = normal_bf16((B, H, Nk, d), seed, 2)
    kl_arr = None if kl is None else np.array(kl, np.int32)
    scale = 1.0 / np.sqrt(d)
    o, lse, guards = run_splitkv(q, k, v, scale, causal, kl_arr, S)
    assert guards, "wrote outside O / LSE"
    o_ref, lse_ref = oracle.attn_ref(q, k, v, scale, causal, kl_arr)
    errs = compare(o, lse, o_ref, lse_ref, str(case))
    print(f"{case}: max|dO|={errs[0]:.3e} relF={errs[1]:.3e} max|dLSE|={errs[2]:.3e}")


@pytest.mark.parametrize("S", [1, 2, 5])
def test_splitkv_agrees_with_single_pass(S):
    # same inputs through both entry points: both are within the oracle bar, and
    # within twice the bar of each other
    B, H, Nq, Nk, d = 2, 3, 130, 1500, 64
    q = normal_bf16((B, H, Nq, d), 71, 0)
    k = normal_bf16((B, H, Nk, d), 71, 1)
    v = normal_bf16((B, H, Nk, d), 71, 2)
    o1, l1 = run_fa(q, k, v, 0.125, True, None)
    o2, l2, _ = run_splitkv(q, k, v, 0.125, True, None, S)
    assert np.abs(o1 - o2).max() <= 3e-2
    assert np.abs(l1 - l2).max() <= 2e-3


def test_splitkv_decode_workload_sampled():
    # decode_16k_d128 at full size: the oracle evaluates every row (there are only B*H of them)
    w = DECODE_WORKLOADS["decode_16k_d128"]
    x = make_inputs(w)
    o, lse, _ = run_splitkv(x["q"], x["k"], x["v"], w.scale, w.causal, x["key_lens"], "auto")
    o_ref, lse_ref = oracle.attn_ref(x["q"], x["k"], x["v"], w.scale, w.causal, x["key_lens"])
    errs = compare(o, lse, o_ref, lse_ref, w.name)
    print(f"{w.name}: max|dO|={errs[0]:.3e} relF={errs[1]:.3e} max|dLSE|={errs[2]:.3e}")


def test_splitkv_deterministic_bitwise():
    B, H, Nq, Nk, d = 1, 4, 2, 5000, 128
    q = normal_bf16((B, H, Nq, d), 72, 0)
    k = normal_bf16((B, H, Nk, d), 72, 1)
    v = normal_bf16((B, H, Nk, d), 72, 2)
    a = run_splitkv(q, k, v, 0.09, False, None, 9)
    b = run_splitkv(q, k, v, 0.09, False, None, 9)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_splitkv_decode_64k_h8_benched_split():
    # decode_64k_h8_d128 at full size, in the configuration bench.py times: the
    # heuristic splits it (8 query blocks cannot fill the GPU), every row compared
    from io_aware_exact_24_b200 import fa_splitkv_num_splits
    w = DECODE_WORKLOADS["decode_64k_h8_d128"]
    ns = fa_splitkv_num_splits(w.B, w.H, w.Nq, w.Nk)
    assert ns > 1
    x = make_inputs(w)
    o, lse, guards = run_splitkv(x["q"], x["k"], x["v"], w.scale, w.causal, x["key_lens"], "auto")
    assert guards, "wrote outside O / LSE"
    o_ref, lse_ref = oracle.attn_ref(x["q"], x["k"], x["v"], w.scale, w.causal, x["key_lens"])
    errs = compare(o, lse, o_ref, lse_ref, w.name)
    print(f"{w.name} ({ns} ranges): max|dO|={errs[0]:.3e} relF={errs[1]:.3e} "
          f"max|dLSE|={errs[2]:.3e}")


@pytest.mark.parametrize("S,d,causal", [(2, 64, False), (37, 128, False), (256, 64, True),
                                        (97, 128, True)])
def test_splitkv_forced_many_ranges_long_keys(S, d, causal):
    # N_k >= 32K with a ragged tail (313 K/V tiles), cut into up to 256 ranges of
    # one or two tiles; a few query rows per head (causal: the last rows, which see
    # nearly every key)
    B, H, Nq, Nk = 1, 3, 3, 40000
    seed = 900 + S + d
    q = normal_bf16((B, H, Nq, d), seed, 0)
    k = normal_bf16((B, H, Nk, d), seed, 1)
    v = normal_bf16((B, H, Nk, d), seed, 2)
    scale = 1.0 / np.sqrt(d)
    o, lse, guards = run_splitkv(q, k, v, scale, causal, None, S)
    assert guards, "wrote outside O / LSE"
    o_ref, lse_ref = oracle.attn_ref(q, k, v, scale, causal, None)
    compare(o, lse, o_ref, lse_ref, f"S={S} d={d} causal={causal}")


@pytest.mark.parametrize("S,d,causal,kl", [(1, 128, False, None), (1, 64, True, [31000, 7]),
                                           (37, 128, True, [40000, 129]), (256, 64, False, [39999, 40000]),
                                           (5, 64, False, [0, 300])])
def test_splitkv_single_row_long_keys(S, d, causal, kl):
    # one query row per head (the decode kernel): N_k = 40000 with a ragged tail,
    # key lengths that end inside a tile, on a tile boundary, or at 0
    B, H, Nq, Nk = 2, 3, 1, 40000
    seed = 950 + S + d
    q = normal_bf16((B, H, Nq, d), seed, 0)
    k = normal_bf16((B, H, Nk, d), seed, 1)
    v = normal_bf16((B, H, Nk, d), seed, 2)
    scale = 1.0 / np.sqrt(d)
    kl_arr = None if kl is None else np.array(kl, np.int32)
    o, lse, guards = run_splitkv(q, k, v, scale, causal, kl_arr, S)
    assert guards, "wrote outside O / LSE"
    o_ref, lse_ref = oracle.attn_ref(q, k, v, scale, causal, kl_arr)
    compare(o, lse, o_ref, lse_ref, f"S={S} d={d} causal={causal} kl={kl}")


def test_splitkv_num_splits_uses_the_device_sm_count():
    import torch
    from io_aware_exact_24_b200 import fa_splitkv_num_splits
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    # one query row, one head and a million keys: one range per SM
    assert fa_splitkv_num_splits(1, 1, 1, 1 << 20) == min(sms, 256)
