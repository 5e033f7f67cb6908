"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the same seeded inputs.

All five workloads are compared element by element over every output row at
their full sizes (the two long ones cost the oracle about half a minute each
on the host cores), plus properties that hold at any size.
"""
import numpy as np
import pytest

import oracle
from io_aware_exact_24_b200.inputs import (WORKLOADS, bf16_bits_to_f32, f32_to_bf16_bits,
                                           make_inputs, normal_bf16)

from fa_testutil import compare, run_fa

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from io_aware_exact_24_b200.build import build
    build()


def _rand(B, H, Nq, Nk, d, seed, sigma=1.0):
    return (normal_bf16((B, H, Nq, d), seed, 0, sigma), normal_bf16((B, H, Nk, d), seed, 1, sigma),
            normal_bf16((B, H, Nk, d), seed, 2, sigma))


@pytest.mark.parametrize("name", ["tiny", "gpt2_causal_1k", "bert_padded_512"])
def test_workload_full_compare(name):
    w = WORKLOADS[name]
    x = make_inputs(w)
    o, lse = run_fa(x["q"], x["k"], x["v"], w.scale, w.causal, x["key_lens"])
    o_ref, lse_ref = oracle.attn_ref(x["q"], x["k"], x["v"], w.scale, w.causal, x["key_lens"])
    errs = compare(o, lse, o_ref, lse_ref, name)
    print(f"{name}: max|dO|={errs[0]:.3e} relF={errs[1]:.3e} max|dLSE|={errs[2]:.3e}")


@pytest.mark.parametrize("name", ["long_16k_d64", "causal_8000_d128"])
def test_workload_full_size_every_row(name):
    # the two long workloads at full size, in the launch configuration bench.py
    # times, against the oracle on every row (per-row S and P keep host memory bounded)
    w = WORKLOADS[name]
    x = make_inputs(w)
    o, lse = run_fa(x["q"], x["k"], x["v"], w.scale, w.causal, x["key_lens"])
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    o_ref, lse_ref = oracle.attn_ref(x["q"], x["k"], x["v"], w.scale, w.causal, x["key_lens"])
    errs = compare(o, lse, o_ref, lse_ref, name)
    print(f"{name} (all {w.B * w.H * w.Nq} rows): max|dO|={errs[0]:.3e} relF={errs[1]:.3e} "
          f"max|dLSE|={errs[2]:.3e}")
    # per (b, h) as well: no head may hide a larger relative error inside the total
    num = np.linalg.norm((o - o_ref).reshape(w.B * w.H, -1), axis=1)
    den = np.linalg.norm(o_ref.reshape(w.B * w.H, -1), axis=1)
    assert (num / den).max() <= 4e-3
    # |O| is bounded by max|V| (each row is a convex combination of V rows)
    vmax = np.abs(bf16_bits_to_f32(x["v"])).max()
    assert np.abs(o).max() <= vmax * (1 + 2**-7)


EDGE = [
    # B, H, Nq, Nk, d, causal, key_lens
    (1, 1, 1, 1, 64, False, None),
    (1, 1, 1, 1, 128, True, None),
    (1, 2, 2, 2, 64, True, None),
    (1, 1, 63, 63, 64, False, None),
    (1, 1, 64, 64, 128, True, None),
    (2, 1, 127, 127, 64, True, None),
    (1, 1, 129, 129, 128, False, None),
    (1, 2, 255, 255, 64, True, None),
    (1, 1, 256, 256, 128, True, None),
    (1, 1, 257, 257, 64, True, None),
    (2, 2, 300, 300, 128, False, None),
    (1, 1, 100, 300, 64, True, None),      # Nq < Nk: bottom-right causal
    (1, 1, 300, 100, 128, True, None),     # Nq > Nk: leading rows see no key
    (1, 1, 513, 129, 64, True, None),      # whole Q tiles with no visible key
    (1, 3, 200, 333, 64, False, None),
    (3, 2, 140, 140, 64, False, [0, 1, 140]),
    (4, 1, 260, 260, 128, True, [0, 129, 1000, -5]),
    (2, 2, 384, 384, 64, False, [128, 255]),
    (1, 1, 64, 0, 64, False, None),        # no keys at all
    (2, 1, 200, 0, 128, True, None),
    (2, 3, 1000, 1000, 128, True, None),   # several tiles, ragged tail
    (1, 2, 1100, 900, 64, False, [700]),
]


@pytest.mark.parametrize("case", EDGE, ids=[str(c[:6]) + ("kl" if c[6] else "") for c in EDGE])
def test_edge_cases(case):
    B, H, Nq, Nk, d, causal, kl = case
    q, k, v = _rand(B, H, Nq, Nk, d, 31 + Nq + Nk + d)
    kl_arr = None if kl is None else np.array(kl, np.int32)
    out = {}
    o, lse = run_fa(q, k, v, 1.0 / np.sqrt(d), causal, kl_arr, o_guard=4096, out=out)
    assert out["guards_ok"], "wrote outside O / LSE"
    o_ref, lse_ref = oracle.attn_ref(q, k, v, 1.0 / np.sqrt(d), causal, kl_arr)
    compare(o, lse, o_ref, lse_ref, str(case))


MANY_BLOCKS = [
    # grids several times the SM count: a running CTA takes over blocks that
    # have not started (B, H, Nq, Nk, d, causal, key_lens)
    (3, 40, 700, 700, 64, True, [700, 0, 333]),
    (2, 48, 520, 600, 128, False, [600, 77]),
    (4, 30, 1000, 1000, 128, True, None),
]


@pytest.mark.parametrize("case", MANY_BLOCKS, ids=[str(c[:6]) for c in MANY_BLOCKS])
def test_more_blocks_than_sms(case):
    B, H, Nq, Nk, d, causal, kl = case
    q, k, v = _rand(B, H, Nq, Nk, d, 91 + Nq + d)
    kl_arr = None if kl is None else np.array(kl, np.int32)
    out = {}
    o, lse = run_fa(q, k, v, 1.0 / np.sqrt(d), causal, kl_arr, o_guard=4096, out=out)
    assert out["guards_ok"], "wrote outside O / LSE"
    o_ref, lse_ref = oracle.attn_ref(q, k, v, 1.0 / np.sqrt(d), causal, kl_arr)
    compare(o, lse, o_ref, lse_ref, str(case))


def test_empty_problems_touch_nothing():
    import torch
    from io_aware_exact_24_b200 import fa_fwd
    o = torch.full((4,), 3.0, dtype=torch.bfloat16, device="cuda")
    lse = torch.full((4,), 5.0, dtype=torch.float32, device="cuda")
    for B, H, Nq in ((0, 2, 8), (2, 0, 8), (2, 2, 0)):
        fa_fwd(o, o, o, o, lse, B, H, Nq, 8, 64, 0.125)
    torch.cuda.synchronize()
    assert (o == 3.0).all() and (lse == 5.0).all()


def test_deterministic_bitwise():
    q, k, v = _rand(2, 4, 700, 700, 128, 77)
    a, b = {}, {}
    run_fa(q, k, v, 0.09, True, None, out=a)
    run_fa(q, k, v, 0.09, True, None, out=b)
    assert np.array_equal(a["o_bits"], b["o_bits"])
    assert np.array_equal(a["lse_raw"].view(np.uint32), b["lse_raw"].view(np.uint32))


def test_masked_garbage_is_invisible_bitwise():
    B, H, N, d = 2, 2, 400, 64
    q, k, v = _rand(B, H, N, N, d, 78)
    kl = np.array([150, 333], np.int32)
    a, b = {}, {}
    run_fa(q, k, v, 0.125, True, kl, out=a)
    k2, v2 = k.copy(), v.copy()
    for bb in range(B):
        k2[bb, :, kl[bb]:] = f32_to_bf16_bits(np.float32(8192.0))
        v2[bb, :, kl[bb]:] = f32_to_bf16_bits(np.float32(-8192.0))
    run_fa(q, k2, v2, 0.125, True, kl, out=b)
    assert np.array_equal(a["o_bits"], b["o_bits"])
    assert np.array_equal(a["lse_raw"].view(np.uint32), b["lse_raw"].view(np.uint32))


def test_single_visible_key_is_exact():
    # causal row 0 and a key_len of 1 see one key: P = 1 exactly, O = V_0 bit for bit
    B, H, N, d = 2, 2, 300, 128
    q, k, v = _rand(B, H, N, N, d, 79)
    o, _ = run_fa(q, k, v, 0.1, True, None)
    vf = bf16_bits_to_f32(v).astype(np.float64)
    assert np.array_equal(o[:, :, 0, :], vf[:, :, 0, :])
    o1, _ = run_fa(q, k, v, 0.1, False, np.array([1, 1], np.int32))
    assert np.array_equal(o1, np.broadcast_to(vf[:, :, :1, :], o1.shape))


def test_zero_query_gives_mean_of_values():
    B, H, N, d = 1, 2, 520, 64
    _, k, v = _rand(B, H, N, N, d, 80)
    q = np.zeros((B, H, N, d), np.uint16)
    o, lse = run_fa(q, k, v, 0.125, True, None)
    vf = bf16_bits_to_f32(v).astype(np.float64)
    means = np.cumsum(vf, axis=2) / np.arange(1, N + 1)[None, None, :, None]
    np.testing.assert_allclose(o, means, rtol=0, atol=1.5e-2)
    np.testing.assert_allclose(lse, np.log(np.arange(1, N + 1))[None, None, :].repeat(H, 1),
                               rtol=0, atol=1e-3)


@pytest.mark.parametrize("shape", [(2, 3, 333, 257, 128, True), (2, 20, 300, 300, 64, False),
                                   (1, 64, 130, 200, 64, True), (40, 2, 200, 150, 64, True)],
                         ids=["heads-6-chunks", "heads-5-per-chunk-tail-3-1-1", "heads-8-per-chunk-tail-4-2-1-1",
                              "whole-batches"])
def test_host_entry_matches_device_entry(shape):
    # the host entry copies and computes in chunks of heads (or of whole batch
    # entries when a batch entry is small), the last chunk of heads cut into
    # halves; every chunk is its own launch, and the result must be the device
    # entry's, bit for bit
    import torch
    from io_aware_exact_24_b200 import fa_fwd_host, fa_fwd_host_workspace_size
    B, H, Nq, Nk, d, with_kl = shape
    q, k, v = _rand(B, H, Nq, Nk, d, 81 + B + H)
    kl = np.array([(Nk * (i + 1)) // B for i in range(B)], np.int32) if with_kl else None
    if with_kl:
        kl[0] = max(1, Nk - 57)
    dev = {}
    run_fa(q, k, v, 0.088, True, kl, out=dev)
    ws_bytes = fa_fwd_host_workspace_size(B, H, Nq, Nk, d, with_kl)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    o = np.empty((B, H, Nq, d), np.uint16)
    lse = np.empty((B, H, Nq), np.float32)
    fa_fwd_host(q, k, v, o, lse, B, H, Nq, Nk, d, 0.088, True, kl, ws, ws_bytes)
    assert np.array_equal(o.view(np.int16), dev["o_bits"])
    assert np.array_equal(lse.view(np.uint32), dev["lse_raw"].view(np.uint32))


def test_device_status_is_clean_after_the_suite():
    from io_aware_exact_24_b200 import FA_OK, fa_get_device_status
    assert fa_get_device_status() == FA_OK


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_rescale_path_with_growing_scores(d, causal):
    # keys grow along the sequence, so most rows move their reference max by more
    # than 2^8 many times: every O-rescale step (including the last tile) runs
    B, H, N = 1, 2, 1100
    q, k, v = _rand(B, H, N, N, d, 90 + d)
    ramp = (1.0 + np.arange(N, dtype=np.float32) / 96.0)[None, None, :, None]
    k = f32_to_bf16_bits(bf16_bits_to_f32(k) * ramp)
    # one very large score in the last key tile of every row
    k[:, :, N - 3, :] = f32_to_bf16_bits(bf16_bits_to_f32(k[:, :, N - 3, :]) * 4.0)
    o, lse = run_fa(q, k, v, 0.5, causal, None)
    o_ref, lse_ref = oracle.attn_ref(q, k, v, 0.5, causal, None)
    compare(o, lse, o_ref, lse_ref, f"growing d{d} causal={causal}")
