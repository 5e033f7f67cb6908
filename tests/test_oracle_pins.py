"""Pins for the fp64 CPU oracle: things the mathematics fixes, checked without the oracle's own code.

Each test below would fail for a plausible slip in the oracle (dropped scale,
wrong sign, transposed operand, off-by-one in a mask, wrong normaliser):

* rows of the materialised P sum to one (softmax normalisation);
* the online-softmax formulation agrees with the two-pass one (the pages
  state the tiled/online result is identical, only the order differs --
  "FlashAttention：把注意力从公式写成数据流", section "分块与在线 softmax");
* closed forms: Q = 0 gives the mean of the visible V rows and LSE = ln|J|;
  a single visible key gives that key's V row and LSE = scale*q.k;
* invariances: constant V column, key shift, joint K/V permutation, garbage
  at masked positions, a dominant score;
* a library routine the special case reduces to: torch's CPU
  scaled_dot_product_attention in float64 with an explicit boolean mask.
"""
import math

import numpy as np
import pytest

import oracle
from io_aware_exact_24_b200.inputs import bf16_bits_to_f32, f32_to_bf16_bits, normal_bf16

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _rand(B, H, Nq, Nk, d, seed, sigma=1.0):
    q = normal_bf16((B, H, Nq, d), seed, 0, sigma)
    k = normal_bf16((B, H, Nk, d), seed, 1, sigma)
    v = normal_bf16((B, H, Nk, d), seed, 2, sigma)
    return q, k, v


def _bits(x):
    """Exactly-representable float values -> bf16 bits (asserts exactness)."""
    x = np.asarray(x, np.float32)
    b = f32_to_bf16_bits(x)
    assert np.array_equal(bf16_bits_to_f32(b), x), "value not exact in bf16"
    return b


def _visible(Nq, Nk, causal, kl):
    """Boolean [Nq, Nk] visibility written from the documented reading."""
    i = np.arange(Nq)[:, None]
    j = np.arange(Nk)[None, :]
    vis = np.broadcast_to(j < kl, (Nq, Nk))
    if causal:
        vis = vis & (j <= i + (Nk - Nq))
    return vis


CASES = [
    # B, H, Nq, Nk, d, causal, key_lens
    (2, 3, 37, 53, 16, False, None),
    (2, 3, 53, 37, 16, True, None),      # Nq > Nk: leading rows fully masked
    (2, 2, 41, 41, 8, True, None),
    (3, 2, 29, 45, 16, False, [0, 17, 45]),
    (3, 2, 45, 45, 16, True, [5, 45, 60]),  # key_len beyond Nk clamps
    (1, 1, 1, 1, 4, False, None),
    (1, 2, 5, 0, 8, False, None),           # no keys at all
]


@pytest.mark.parametrize("case", CASES)
def test_p_rows_sum_to_one(case):
    B, H, Nq, Nk, d, causal, kl = case
    q, k, v = _rand(B, H, Nq, Nk, d, 11)
    kl_arr = None if kl is None else np.array(kl, np.int32)
    o, lse, p = oracle.attn_ref(q, k, v, 0.25, causal, kl_arr, return_p=True)
    for b in range(B):
        klb = Nk if kl is None else min(max(kl[b], 0), Nk)
        vis = _visible(Nq, Nk, causal, klb)
        for h in range(H):
            sums = p[b, h].sum(axis=1)
            has = vis.any(axis=1)
            np.testing.assert_allclose(sums[has], 1.0, rtol=0, atol=1e-12)
            assert np.all(p[b, h][~vis] == 0.0)
            assert np.all(np.isneginf(lse[b, h][~has]))
            assert np.all(o[b, h][~has] == 0.0)


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("block", [1, 7, 128])
def test_online_matches_two_pass(case, block):
    B, H, Nq, Nk, d, causal, kl = case
    q, k, v = _rand(B, H, Nq, Nk, d, 12)
    kl_arr = None if kl is None else np.array(kl, np.int32)
    o1, l1 = oracle.attn_ref(q, k, v, 0.3, causal, kl_arr)
    o2, l2 = oracle.attn_online(q, k, v, 0.3, causal, kl_arr, block=block)
    np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-12)
    fin = np.isfinite(l1)
    assert np.array_equal(fin, np.isfinite(l2))
    np.testing.assert_allclose(l2[fin], l1[fin], rtol=1e-12, atol=1e-12)


def test_online_matches_two_pass_tiny_workload():
    from io_aware_exact_24_b200.inputs import WORKLOADS, make_inputs
    w = WORKLOADS["tiny"]
    x = make_inputs(w)
    o1, l1 = oracle.attn_ref(x["q"], x["k"], x["v"], w.scale, w.causal, x["key_lens"])
    o2, l2 = oracle.attn_online(x["q"], x["k"], x["v"], w.scale, w.causal, x["key_lens"])
    np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l2, l1, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("causal,kl", [(False, None), (True, None), (False, [7, 30]),
                                       (True, [3, 30])])
def test_zero_query_gives_mean_of_visible_values(causal, kl):
    B, H, Nq, Nk, d = 2, 2, 24, 30, 8
    _, k, v = _rand(B, H, Nq, Nk, d, 13)
    q = np.zeros((B, H, Nq, d), np.uint16)          # +0.0 in bf16
    kl_arr = None if kl is None else np.array(kl, np.int32)
    o, lse = oracle.attn_ref(q, k, v, 0.7, causal, kl_arr)
    vf = bf16_bits_to_f32(v).astype(np.float64)
    for b in range(B):
        vis = _visible(Nq, Nk, causal, Nk if kl is None else kl[b])
        for h in range(H):
            for i in range(Nq):
                n = int(vis[i].sum())
                if n == 0:
                    assert np.all(o[b, h, i] == 0) and np.isneginf(lse[b, h, i])
                    continue
                np.testing.assert_allclose(o[b, h, i], vf[b, h, vis[i]].mean(axis=0),
                                           rtol=0, atol=1e-13)
                assert abs(lse[b, h, i] - math.log(n)) < 1e-13


def test_single_key_returns_its_value_row():
    B, H, Nq, d = 2, 3, 9, 16
    q, k, v = _rand(B, H, Nq, 1, d, 14)
    o, lse = oracle.attn_ref(q, k, v, 0.125)
    qf = bf16_bits_to_f32(q).astype(np.float64)
    kf = bf16_bits_to_f32(k).astype(np.float64)
    vf = bf16_bits_to_f32(v).astype(np.float64)
    assert np.array_equal(o, np.broadcast_to(vf, o.shape))      # exact: P = 1
    dots = np.einsum("bhid,bhjd->bhij", qf, kf)[..., 0]
    np.testing.assert_allclose(lse, 0.125 * dots, rtol=1e-14, atol=1e-14)


def test_causal_first_row_sees_only_first_key():
    B, H, N, d = 1, 4, 33, 16
    q, k, v = _rand(B, H, N, N, d, 15)
    o, lse = oracle.attn_ref(q, k, v, 0.125, causal=True)
    vf = bf16_bits_to_f32(v).astype(np.float64)
    assert np.array_equal(o[:, :, 0, :], vf[:, :, 0, :])


def test_constant_value_column_is_reproduced():
    B, H, Nq, Nk, d = 2, 2, 17, 40, 8
    q, k, v = _rand(B, H, Nq, Nk, d, 16)
    v = v.copy()
    v[..., 3] = _bits(1.5)
    v[..., 5] = _bits(-0.375)
    for causal, kl in ((False, None), (True, np.array([40, 9], np.int32))):
        o, _ = oracle.attn_ref(q, k, v, 0.2, causal, kl)
        np.testing.assert_allclose(o[..., 3], 1.5, rtol=0, atol=1e-14)
        np.testing.assert_allclose(o[..., 5], -0.375, rtol=0, atol=1e-14)


def test_key_shift_leaves_output_and_moves_lse():
    # small integers: every sum stays exact in bf16 and fp64
    rng = np.random.default_rng(0)
    B, H, Nq, Nk, d = 1, 2, 12, 20, 4
    qv = rng.integers(-2, 3, size=(B, H, Nq, d)).astype(np.float32)
    kv = rng.integers(-2, 3, size=(B, H, Nk, d)).astype(np.float32)
    vv = rng.integers(-4, 5, size=(B, H, Nk, d)).astype(np.float32)
    w = np.array([1, -2, 0, 3], np.float32)
    scale = 0.25
    o1, l1 = oracle.attn_ref(_bits(qv), _bits(kv), _bits(vv), scale, causal=True)
    o2, l2 = oracle.attn_ref(_bits(qv), _bits(kv + w), _bits(vv), scale, causal=True)
    np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-13)
    shift = scale * (qv.astype(np.float64) @ w.astype(np.float64))
    np.testing.assert_allclose(l2 - l1, shift, rtol=0, atol=1e-12)


def test_joint_key_value_permutation_and_query_permutation():
    B, H, Nq, Nk, d = 1, 2, 19, 31, 16
    q, k, v = _rand(B, H, Nq, Nk, d, 17)
    o1, l1 = oracle.attn_ref(q, k, v, 0.125)
    perm = np.random.default_rng(1).permutation(Nk)
    o2, l2 = oracle.attn_ref(q, k[:, :, perm], v[:, :, perm], 0.125)
    np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l2, l1, rtol=0, atol=1e-13)
    qperm = np.random.default_rng(2).permutation(Nq)
    o3, l3 = oracle.attn_ref(q[:, :, qperm], k, v, 0.125)
    assert np.array_equal(o3, o1[:, :, qperm]) and np.array_equal(l3, l1[:, :, qperm])


def test_masked_positions_never_contribute():
    B, H, Nq, Nk, d = 2, 2, 40, 40, 16
    q, k, v = _rand(B, H, Nq, Nk, d, 18)
    kl = np.array([25, 33], np.int32)
    o1, l1 = oracle.attn_ref(q, k, v, 0.125, True, kl)
    k2, v2 = k.copy(), v.copy()
    garbage = _bits(np.float32(8192.0))
    for b in range(B):
        k2[b, :, kl[b]:] = garbage
        v2[b, :, kl[b]:] = _bits(np.float32(-8192.0))
    o2, l2 = oracle.attn_ref(q, k2, v2, 0.125, True, kl)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
    o3, l3 = oracle.attn_online(q, k2, v2, 0.125, True, kl)
    np.testing.assert_allclose(o3, o1, rtol=0, atol=1e-12)


def test_dominant_score_selects_its_value_row():
    B, H, Nq, Nk, d = 1, 1, 3, 16, 4
    q = np.zeros((B, H, Nq, d), np.float32)
    q[..., 0] = 1.0
    k = np.zeros((B, H, Nk, d), np.float32)
    k[0, 0, 5, 0] = 100.0                       # score 100 above every other
    v = np.random.default_rng(3).integers(-3, 4, size=(B, H, Nk, d)).astype(np.float32)
    o, lse = oracle.attn_ref(_bits(q), _bits(k), _bits(v), 1.0)
    np.testing.assert_allclose(o[0, 0], np.broadcast_to(v[0, 0, 5], (Nq, d)), rtol=0,
                               atol=1e-40 + 20 * math.exp(-100) * 4)
    np.testing.assert_allclose(lse, 100.0 + math.log1p(15 * math.exp(-100)), rtol=0,
                               atol=1e-13)


@pytest.mark.parametrize("case", CASES[:5])
def test_matches_torch_sdpa_float64(case):
    torch = pytest.importorskip("torch")
    import torch.nn.functional as F
    B, H, Nq, Nk, d, causal, kl = case
    q, k, v = _rand(B, H, Nq, Nk, d, 19)
    kl_arr = None if kl is None else np.array(kl, np.int32)
    scale = 0.2
    o, lse = oracle.attn_ref(q, k, v, scale, causal, kl_arr)
    tq, tk, tv = (torch.from_numpy(bf16_bits_to_f32(x).astype(np.float64)) for x in (q, k, v))
    mask = np.zeros((B, 1, Nq, Nk), bool)
    for b in range(B):
        mask[b, 0] = _visible(Nq, Nk, causal, Nk if kl is None else kl[b])
    tmask = torch.from_numpy(mask)
    ref = F.scaled_dot_product_attention(tq, tk, tv, attn_mask=tmask,
                                         scale=float(np.float32(scale))).numpy()
    scores = torch.einsum("bhid,bhjd->bhij", tq, tk) * float(np.float32(scale))
    ref_lse = torch.logsumexp(scores.masked_fill(~tmask, float("-inf")), dim=-1).numpy()
    has = np.broadcast_to(mask.any(axis=-1), (B, H, Nq))
    np.testing.assert_allclose(o[has], ref[has], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse[has], ref_lse[has], rtol=0, atol=1e-12)


def test_rows_entry_matches_full_evaluation():
    B, H, Nq, Nk, d = 2, 3, 21, 34, 16
    q, k, v = _rand(B, H, Nq, Nk, d, 20)
    kl = np.array([34, 11], np.int32)
    o, lse = oracle.attn_ref(q, k, v, 0.125, True, kl)
    rows = np.array([0, 5, 20, 21, 63, 64, B * H * Nq - 1], np.int64)
    orow, lrow = oracle.attn_ref_rows(q, k, v, 0.125, rows, True, kl)
    assert np.array_equal(orow, o.reshape(-1, d)[rows])
    assert np.array_equal(lrow, lse.reshape(-1)[rows])


# ---------------------------------------------------------------- sliding window

WINDOW_CASES = [
    # B, H, Nq, Nk, d, causal, key_lens, W
    (1, 2, 9, 9, 8, True, None, 3),
    (2, 1, 7, 12, 16, True, [12, 5], 2),
    (1, 1, 12, 5, 8, True, None, 1),      # N_q > N_k: leading rows see nothing
    (2, 2, 6, 10, 8, False, [3, 10], 4),  # non-causal: only the lower bound applies
    (1, 1, 16, 16, 4, True, None, 0),
]


def _window_rows(Nq, Nk, causal, kl, W):
    lo = [max(0, i + Nk - Nq - W) for i in range(Nq)]
    hi = [min(kl, i + Nk - Nq + 1) if causal else kl for i in range(Nq)]
    return lo, [max(h, 0) for h in hi]


@pytest.mark.parametrize("case", WINDOW_CASES)
def test_window_equals_plain_attention_on_the_key_slice(case):
    # a window only removes keys: each row equals the plain (unmasked) definition
    # evaluated on its own slice [lo, hi) of K and V
    B, H, Nq, Nk, d, causal, kl, W = case
    q, k, v = _rand(B, H, Nq, Nk, d, 31)
    kl_arr = None if kl is None else np.array(kl, np.int32)
    o, lse = oracle.attn_ref_window(q, k, v, 0.3, W, causal, kl_arr)
    for b in range(B):
        lo, hi = _window_rows(Nq, Nk, causal, Nk if kl is None else kl[b], W)
        for h in range(H):
            for i in range(Nq):
                if hi[i] <= lo[i]:
                    assert np.all(o[b, h, i] == 0) and np.isneginf(lse[b, h, i])
                    continue
                sl = slice(lo[i], hi[i])
                o1, l1 = oracle.attn_ref(q[b:b + 1, h:h + 1, i:i + 1], k[b:b + 1, h:h + 1, sl],
                                         v[b:b + 1, h:h + 1, sl], 0.3, False, None)
                np.testing.assert_allclose(o[b, h, i], o1[0, 0, 0], rtol=0, atol=1e-13)
                assert abs(lse[b, h, i] - l1[0, 0, 0]) <= 1e-13


def test_window_zero_sees_only_the_diagonal_key():
    # W = 0 with causal and N_q = N_k: row i sees key i alone, so O_i = V_i and
    # LSE_i = scale * q_i . k_i exactly (closed form)
    q, k, v = _rand(2, 2, 11, 11, 8, 32)
    o, lse = oracle.attn_ref_window(q, k, v, 0.25, 0, True, None)
    qf, kf, vf = (bf16_bits_to_f32(x).astype(np.float64) for x in (q, k, v))
    assert np.array_equal(o, vf)
    s_diag = np.einsum("bhid,bhid->bhi", qf, kf) * float(np.float32(0.25))
    np.testing.assert_allclose(lse, s_diag, rtol=0, atol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_wide_window_is_no_window(causal):
    q, k, v = _rand(2, 3, 13, 17, 8, 33)
    kl = np.array([17, 9], np.int32)
    o0, l0 = oracle.attn_ref(q, k, v, 0.2, causal, kl)
    for W in (17, 40):
        o1, l1 = oracle.attn_ref_window(q, k, v, 0.2, W, causal, kl)
        assert np.array_equal(o0, o1) and np.array_equal(l0, l1)
    o2, l2 = oracle.attn_ref_window(q, k, v, 0.2, -1, causal, kl)
    assert np.array_equal(o0, o2) and np.array_equal(l0, l2)


# ---------------------------------------------------------------- additive positional bias

def test_zero_slopes_are_no_bias():
    q, k, v = _rand(2, 3, 9, 14, 8, 34)
    kl = np.array([14, 6], np.int32)
    for causal in (False, True):
        o0, l0 = oracle.attn_ref(q, k, v, 0.2, causal, kl)
        o1, l1 = oracle.attn_ref_bias(q, k, v, 0.2, np.zeros(3, np.float32), causal, kl)
        assert np.array_equal(o0, o1) and np.array_equal(l0, l1)


def test_bias_with_zero_query_is_a_geometric_weighting():
    # q = 0: scores are the bias alone, -m*(pos - j) for j <= pos (causal), so
    # LSE = ln sum_{t=0}^{pos} e^{-m t} = ln((1 - e^{-m(pos+1)}) / (1 - e^{-m}))
    # and O is the e^{-m(pos-j)}-weighted mean of the visible value rows
    B, H, N, d = 1, 2, 13, 8
    _, k, v = _rand(B, H, N, N, d, 35)
    q = np.zeros((B, H, N, d), np.uint16)
    slopes = np.array([0.5, 0.0625], np.float32)
    o, lse = oracle.attn_ref_bias(q, k, v, 0.3, slopes, True, None)
    vf = bf16_bits_to_f32(v).astype(np.float64)
    for h in range(H):
        m = float(slopes[h])
        for i in range(N):
            closed = math.log((1 - math.exp(-m * (i + 1))) / (1 - math.exp(-m)))
            assert abs(lse[0, h, i] - closed) <= 1e-12
            w = np.exp(-m * (i - np.arange(i + 1)))
            np.testing.assert_allclose(o[0, h, i], (w[:, None] * vf[0, h, :i + 1]).sum(0) / w.sum(),
                                       rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal,W", [(True, -1), (False, -1), (True, 5)])
def test_bias_matches_torch_sdpa_with_an_additive_mask(causal, W):
    torch = pytest.importorskip("torch")
    import torch.nn.functional as F
    B, H, Nq, Nk, d = 2, 2, 11, 17, 8
    q, k, v = _rand(B, H, Nq, Nk, d, 36)
    kl = np.array([17, 9], np.int32)
    slopes = np.array([0.25, 0.03125], np.float32)
    scale = 0.2
    o, lse = oracle.attn_ref_bias(q, k, v, scale, slopes, causal, kl, W)
    tq, tk, tv = (torch.from_numpy(bf16_bits_to_f32(x).astype(np.float64)) for x in (q, k, v))
    i = np.arange(Nq)[:, None] + (Nk - Nq)
    j = np.arange(Nk)[None, :]
    bias = np.zeros((B, H, Nq, Nk))
    for b in range(B):
        vis = j < kl[b]
        if causal:
            vis = vis & (j <= i)
        if W >= 0:
            vis = vis & (j >= i - W)
        for h in range(H):
            bias[b, h] = np.where(vis, -float(slopes[h]) * np.abs(i - j), -np.inf)
    tb = torch.from_numpy(bias)
    ref = F.scaled_dot_product_attention(tq, tk, tv, attn_mask=tb,
                                         scale=float(np.float32(scale))).numpy()
    ref_lse = torch.logsumexp(torch.einsum("bhid,bhjd->bhij", tq, tk) * float(np.float32(scale))
                              + tb, dim=-1).numpy()
    has = np.isfinite(ref_lse)
    np.testing.assert_allclose(o[has], ref[has], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse[has], ref_lse[has], rtol=0, atol=1e-12)
    assert np.all(np.isneginf(lse[~has]))


# ---------------------------------------------------------------- custom positional bias table
# "FlashAttention：把注意力从公式写成数据流", section "精度、掩码和边界情况", lists
# custom positional bias among the mask variants.  Reading: a per-head table of
# 2R+1 values indexed by the key's position relative to the query's diagonal
# position, clamped to [-R, R], added to the scaled scores.

def _table(H, R, seed, sigma=1.0):
    return (np.random.default_rng(seed).standard_normal((H, 2 * R + 1)) * sigma).astype(np.float32)


def test_zero_table_is_no_bias():
    q, k, v = _rand(2, 3, 9, 14, 8, 40)
    kl = np.array([14, 6], np.int32)
    for causal, W in ((False, -1), (True, -1), (True, 4)):
        o0, l0 = oracle.attn_ref_window(q, k, v, 0.2, W, causal, kl)
        o1, l1 = oracle.attn_ref_bias_table(q, k, v, 0.2, np.zeros((3, 7), np.float32), causal, kl, W)
        assert np.array_equal(o0, o1) and np.array_equal(l0, l1)


def test_constant_table_shifts_only_the_lse():
    # a constant bias c on every visible score: P and O unchanged, LSE + c
    q, k, v = _rand(1, 2, 10, 12, 8, 41)
    o0, l0 = oracle.attn_ref(q, k, v, 0.3, True)
    c = np.float32(1.75)
    o1, l1 = oracle.attn_ref_bias_table(q, k, v, 0.3, np.full((2, 9), c, np.float32), True)
    np.testing.assert_allclose(o1, o0, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l1, l0 + float(c), rtol=0, atol=1e-13)


def test_table_with_zero_query_is_its_softmax_weighting():
    # q = 0: row i's scores are the table entries of its relative positions alone,
    # so LSE_i = ln sum_j e^{T[clamp(j - i, -R, R) + R]} and O_i is the matching
    # weighted mean of the visible value rows; R = 3 < N makes the clamp matter
    B, H, N, d, R = 1, 2, 11, 8, 3
    _, k, v = _rand(B, H, N, N, d, 42)
    q = np.zeros((B, H, N, d), np.uint16)
    tab = _table(H, R, 43)
    o, lse = oracle.attn_ref_bias_table(q, k, v, 0.3, tab, False, None)
    vf = bf16_bits_to_f32(v).astype(np.float64)
    for h in range(H):
        for i in range(N):
            rel = [min(max(j - i, -R), R) for j in range(N)]
            w = [math.exp(float(tab[h, r + R])) for r in rel]
            assert abs(lse[0, h, i] - math.log(sum(w))) <= 1e-12
            ref = sum(w[j] * vf[0, h, j] for j in range(N)) / sum(w)
            np.testing.assert_allclose(o[0, h, i], ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal,W,R", [(True, -1, 40), (False, -1, 40), (True, 5, 40),
                                        (False, -1, 4), (True, -1, 2)])
def test_bias_table_matches_torch_sdpa_with_an_additive_mask(causal, W, R):
    torch = pytest.importorskip("torch")
    import torch.nn.functional as F
    B, H, Nq, Nk, d = 2, 2, 11, 17, 8
    q, k, v = _rand(B, H, Nq, Nk, d, 44)
    kl = np.array([17, 9], np.int32)
    tab = _table(H, R, 45 + R)
    scale = 0.2
    o, lse = oracle.attn_ref_bias_table(q, k, v, scale, tab, causal, kl, W)
    tq, tk, tv = (torch.from_numpy(bf16_bits_to_f32(x).astype(np.float64)) for x in (q, k, v))
    i = np.arange(Nq)[:, None] + (Nk - Nq)
    j = np.arange(Nk)[None, :]
    idx = np.clip(j - i, -R, R) + R
    bias = np.zeros((B, H, Nq, Nk))
    for b in range(B):
        vis = j < kl[b]
        if causal:
            vis = vis & (j <= i)
        if W >= 0:
            vis = vis & (j >= i - W)
        for h in range(H):
            bias[b, h] = np.where(vis, tab[h][idx].astype(np.float64), -np.inf)
    tb = torch.from_numpy(bias)
    ref = F.scaled_dot_product_attention(tq, tk, tv, attn_mask=tb,
                                         scale=float(np.float32(scale))).numpy()
    ref_lse = torch.logsumexp(torch.einsum("bhid,bhjd->bhij", tq, tk) * float(np.float32(scale))
                              + tb, dim=-1).numpy()
    has = np.isfinite(ref_lse)
    np.testing.assert_allclose(o[has], ref[has], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse[has], ref_lse[has], rtol=0, atol=1e-12)
    assert np.all(np.isneginf(lse[~has]))


def test_bias_table_rejects_an_even_width():
    q, k, v = _rand(1, 2, 4, 4, 8, 46)
    with pytest.raises(ValueError):
        oracle.attn_ref_bias_table(q, k, v, 0.2, np.zeros((2, 6), np.float32))


def test_varlen_of_equal_lengths_is_the_dense_problem():
    # packing B equal-length sequences token-major is a relayout of the dense batch
    B, H, N, d = 3, 2, 9, 8
    q, k, v = _rand(B, H, N, N, d, 37)
    o, lse = oracle.attn_ref(q, k, v, 0.3, True, None)
    pack = lambda x: x.transpose(0, 2, 1, 3).reshape(B * N, H, d)
    cu = np.arange(B + 1) * N
    ov, lv = oracle.attn_ref_varlen(pack(q), pack(k), pack(v), cu, cu, 0.3, True)
    assert np.array_equal(ov, o.transpose(0, 2, 1, 3).reshape(B * N, H, d))
    assert np.array_equal(lv, lse.transpose(0, 2, 1).reshape(B * N, H))


# ---------------------------------------------------------------- e4m3 inputs
# Pins of the FP8 wrapper: the code decode against a library conversion and the
# format's closed forms, and the algebra of the three descales against the
# (already pinned) bf16 oracle on the same values.

def test_e4m3_decode_matches_torch_on_all_codes():
    torch = pytest.importorskip("torch")
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_to_f64(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    fin = ~np.isnan(ref)
    assert np.array_equal(ours[fin], ref[fin])
    assert np.array_equal(np.signbit(ours[fin]), np.signbit(ref[fin]))


def test_e4m3_closed_forms():
    d = oracle.e4m3_to_f64(np.array([0x00, 0x80, 0x38, 0xB8, 0x7E, 0xFE, 0x01, 0x07, 0x08, 0x7F, 0xFF],
                                    np.uint8))
    assert d[0] == 0 and not np.signbit(d[0]) and d[1] == 0 and np.signbit(d[1])
    assert d[2] == 1.0 and d[3] == -1.0
    assert d[4] == 448.0 and d[5] == -448.0          # largest finite: 1.75 * 2^8
    assert d[6] == 2.0 ** -9 and d[7] == 7 * 2.0 ** -9  # subnormals m * 2^-9
    assert d[8] == 2.0 ** -6                          # smallest normal
    assert np.isnan(d[9]) and np.isnan(d[10])
    bits = oracle.e4m3_to_bf16_bits(np.array([0x38, 0x7E, 0x01], np.uint8))
    assert list(bits) == [0x3F80, 0x43E0, 0x3B00]


def _codes(shape, seed):
    rng = np.random.default_rng(seed)
    c = rng.integers(0, 256, size=shape, dtype=np.uint8)
    c[(c & 0x7F) == 0x7F] = 0x38                      # no NaN codes
    return c


@pytest.mark.parametrize("causal,kl", [(False, None), (True, None), (False, [5, 40])])
def test_e4m3_unit_descales_are_the_bf16_oracle(causal, kl):
    B, H, Nq, Nk, d = 2, 2, 33, 40, 16
    q8 = _codes((B, H, Nq, d), 1) & 0xBF              # exponents <= 7: moderate scores
    k8 = _codes((B, H, Nk, d), 2) & 0xBF
    v8 = _codes((B, H, Nk, d), 3)
    kl_arr = None if kl is None else np.array(kl, np.int32)
    o, lse = oracle.attn_ref_e4m3(q8, k8, v8, 0.03125, 1.0, 1.0, 1.0, causal, kl_arr)
    qf, kf, vf = (oracle.e4m3_to_f64(x).astype(np.float32) for x in (q8, k8, v8))
    o2, l2 = oracle.attn_ref(_bits(qf), _bits(kf), _bits(vf), 0.03125, causal, kl_arr)
    assert np.array_equal(o, o2) and np.array_equal(lse, l2)


def test_e4m3_descales_scale_scores_and_values():
    B, H, Nq, Nk, d = 1, 2, 20, 24, 8
    q8 = _codes((B, H, Nq, d), 4) & 0xBF
    k8 = _codes((B, H, Nk, d), 5) & 0xBF
    v8 = _codes((B, H, Nk, d), 6)
    base_o, base_l = oracle.attn_ref_e4m3(q8, k8, v8, 0.02, 1.0, 1.0, 1.0)
    # q and k descales multiply the scores: (2, 0.5) is (1, 1); (2, 1) is scale * 2
    o, lse = oracle.attn_ref_e4m3(q8, k8, v8, 0.02, 2.0, 0.5, 1.0)
    assert np.array_equal(o, base_o) and np.array_equal(lse, base_l)
    o, lse = oracle.attn_ref_e4m3(q8, k8, v8, 0.02, 2.0, 1.0, 1.0)
    o2, l2 = oracle.attn_ref_e4m3(q8, k8, v8, 0.04, 1.0, 1.0, 1.0)
    assert np.array_equal(o, o2) and np.array_equal(lse, l2)
    assert not np.allclose(lse, base_l)
    # the v descale multiplies O and leaves the LSE alone
    o, lse = oracle.attn_ref_e4m3(q8, k8, v8, 0.02, 1.0, 1.0, 0.25)
    assert np.array_equal(o, base_o * 0.25) and np.array_equal(lse, base_l)


def test_e4m3_zero_query_gives_the_scaled_mean_of_values():
    B, H, Nq, Nk, d = 1, 1, 6, 10, 8
    q8 = np.zeros((B, H, Nq, d), np.uint8)
    k8 = _codes((B, H, Nk, d), 7)
    v8 = _codes((B, H, Nk, d), 8)
    o, lse = oracle.attn_ref_e4m3(q8, k8, v8, 0.1, 3.0, 5.0, 0.5, causal=True)
    vf = oracle.e4m3_to_f64(v8)[0, 0]
    for i in range(Nq):
        n = i + (Nk - Nq) + 1
        np.testing.assert_allclose(o[0, 0, i], 0.5 * vf[:n].mean(axis=0), rtol=0, atol=1e-12)
        assert abs(lse[0, 0, i] - math.log(n)) < 1e-13


def test_e4m3_score_factor_is_the_exact_product():
    # One visible key: LSE = scale * qd * kd * (q8 . k8) in closed form, with the
    # product of the three fp32 factors taken exactly (the definition of the
    # dequantised scores), not folded into one fp32 number first.
    d = 8
    q8 = np.array([[[[0x38, 0x40, 0x30, 0xB8, 0x3C, 0x28, 0x44, 0x34]]]], np.uint8)
    k8 = np.array([[[[0x3A, 0xB0, 0x38, 0x2C, 0x40, 0x36, 0xB4, 0x38]]]], np.uint8)
    v8 = np.full((1, 1, 1, d), 0x38, np.uint8)
    scale, qd, kd = 0.1, 1.0 / 3.0, 0.7
    f = lambda x: np.float64(np.float32(x))
    dot = float(oracle.e4m3_to_f64(q8)[0, 0, 0] @ oracle.e4m3_to_f64(k8)[0, 0, 0])
    exact = f(scale) * f(qd) * f(kd) * dot
    folded = float(np.float32(np.float32(np.float32(scale) * np.float32(qd)) * np.float32(kd))) * dot
    assert abs(folded - exact) > 1e-9 * abs(exact)     # the two readings differ here
    _, lse = oracle.attn_ref_e4m3(q8, k8, v8, scale, qd, kd, 1.0)
    assert abs(lse[0, 0, 0] - exact) <= 1e-15 * abs(exact)


def test_e4m3_rows_entry_matches_full_evaluation():
    B, H, Nq, Nk, d = 2, 2, 17, 23, 16
    q8, k8, v8 = _codes((B, H, Nq, d), 9) & 0xBF, _codes((B, H, Nk, d), 10) & 0xBF, _codes((B, H, Nk, d), 11)
    o, lse = oracle.attn_ref_e4m3(q8, k8, v8, 0.05, 1.5, 0.75, 2.0, True)
    rows = np.array([0, 5, 16, 17, 40, 67], np.int64)
    orow, lrow = oracle.attn_ref_rows_e4m3(q8, k8, v8, 0.05, 1.5, 0.75, 2.0, rows, True)
    assert np.array_equal(orow, o.reshape(-1, d)[rows]) and np.array_equal(lrow, lse.reshape(-1)[rows])


# ---------------------------------------------------------------- backward oracle
# Pins of oracle.attn_bwd_ref: a library routine the case reduces to (torch float64
# autograd through its scaled_dot_product_attention with a boolean mask), the
# forward it recomputes equals the pinned forward, and properties fixed by the
# mathematics (softmax-gradient rows sum to zero, key-shift invariance, a closed form).

BWD_CASES = [
    # B, H, Nq, Nk, d, causal, key_lens
    (2, 2, 19, 23, 8, False, None),
    (1, 3, 23, 23, 16, True, None),
    (2, 2, 15, 30, 8, True, None),           # N_q < N_k: bottom-right diagonal
    (2, 1, 17, 21, 8, False, [9, 21]),
]


@pytest.mark.parametrize("case", BWD_CASES, ids=[str(c) for c in BWD_CASES])
def test_bwd_matches_torch_autograd_float64(case):
    torch = pytest.importorskip("torch")
    B, H, Nq, Nk, d, causal, kl = case
    q, k, v = _rand(B, H, Nq, Nk, d, 61)
    do = normal_bf16((B, H, Nq, d), 61, 5)
    kl_arr = None if kl is None else np.array(kl, np.int32)
    scale = 0.37
    dq, dk, dv = oracle.attn_bwd_ref(q, k, v, do, scale, causal, kl_arr)
    tq, tk, tv = (torch.from_numpy(bf16_bits_to_f32(x).astype(np.float64)).requires_grad_(True)
                  for x in (q, k, v))
    tdo = torch.from_numpy(bf16_bits_to_f32(do).astype(np.float64))
    mask = np.stack([_visible(Nq, Nk, causal, Nk if kl is None else kl[b]) for b in range(B)])
    out = torch.nn.functional.scaled_dot_product_attention(
        tq, tk, tv, attn_mask=torch.from_numpy(mask)[:, None], scale=float(np.float32(scale)))
    out.backward(tdo)
    np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=0, atol=1e-11)
    np.testing.assert_allclose(dk, tk.grad.numpy(), rtol=0, atol=1e-11)
    np.testing.assert_allclose(dv, tv.grad.numpy(), rtol=0, atol=1e-11)


def test_bwd_recomputed_forward_is_the_pinned_forward():
    q, k, v = _rand(2, 2, 21, 26, 16, 62)
    do = normal_bf16((2, 2, 21, 16), 62, 5)
    kl = np.array([0, 20], np.int32)
    _, _, _, parts = oracle.attn_bwd_ref(q, k, v, do, 0.25, True, kl, return_parts=True)
    o, _ = oracle.attn_ref(q, k, v, 0.25, True, kl)
    np.testing.assert_allclose(np.stack(parts["O"]).reshape(o.shape), o, rtol=0, atol=1e-13)


def test_bwd_key_gradients_sum_to_zero_and_masked_keys_get_none():
    B, H, Nq, Nk, d = 2, 2, 20, 28, 8
    q, k, v = _rand(B, H, Nq, Nk, d, 63)
    do = normal_bf16((B, H, Nq, d), 63, 5)
    kl = np.array([28, 11], np.int32)
    dq, dk, dv = oracle.attn_bwd_ref(q, k, v, do, 0.3, True, kl)
    # each row of dS sums to zero, so sum_j dK_j = scale * sum_i (sum_j dS_ij) Q_i = 0
    assert np.abs(dk.sum(axis=2)).max() < 1e-12
    # keys past key_len are never visible: no gradient reaches them
    assert np.all(dk[1, :, 11:] == 0) and np.all(dv[1, :, 11:] == 0)


def test_bwd_key_shift_leaves_every_gradient_unchanged():
    B, H, Nq, Nk, d = 1, 2, 12, 16, 8
    rng = np.random.default_rng(64)
    q = _bits(rng.integers(-3, 4, (B, H, Nq, d)).astype(np.float32) / 4)
    k = _bits(rng.integers(-3, 4, (B, H, Nk, d)).astype(np.float32) / 4)
    v = _bits(rng.integers(-3, 4, (B, H, Nk, d)).astype(np.float32) / 4)
    do = _bits(rng.integers(-3, 4, (B, H, Nq, d)).astype(np.float32) / 4)
    w = rng.integers(-2, 3, d).astype(np.float32) / 2
    k2 = _bits(bf16_bits_to_f32(k) + w)
    g1 = oracle.attn_bwd_ref(q, k, v, do, 0.5, True)
    g2 = oracle.attn_bwd_ref(q, k2, v, do, 0.5, True)
    for a, b in zip(g1, g2):
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def test_bwd_zero_query_closed_form_for_dv():
    B, H, Nq, Nk, d = 1, 2, 10, 10, 8
    _, k, v = _rand(B, H, Nq, Nk, d, 65)
    q = np.zeros((B, H, Nq, d), np.uint16)
    do = normal_bf16((B, H, Nq, d), 65, 5)
    _, _, dv = oracle.attn_bwd_ref(q, k, v, do, 0.9, True)
    dof = bf16_bits_to_f32(do).astype(np.float64)
    # P is uniform over keys 0..i: dV_j = sum_{i >= j} dO_i / (i + 1)
    for j in range(Nk):
        ref = sum(dof[0, :, i] / (i + 1) for i in range(j, Nq))
        np.testing.assert_allclose(dv[0, :, j], ref, rtol=0, atol=1e-13)
