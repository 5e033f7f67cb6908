"""GPU parity of the backward pass (``fa_bwd``) against the fp64 oracle
(``oracle.attn_bwd_ref``: the chain rule of the plain definition, exact O and P).

Tolerance, derived element by element from the arithmetic (nothing fitted):
the kernel recomputes P = exp2(S c - LSE log2 e) from the GPU forward's fp32 LSE,
takes D_i = dO_i . O_i from the forward's bf16 O, rounds P and dS to bf16 before
the MMAs, accumulates in fp32 and rounds dQ, dK, dV to bf16.  With n the sum
length and u32 = 2^-23 (generous for tensor-core fp32 sums):
  eP_ij  = |dLSE_i| + d u32 scale sum_c |q_ic k_jc| + 2^-20      (relative error of P)
  dD_i   = sum_c |dO_ic| |O'_ic - O_ic| + d u32 sum_c |dO_ic O_ic|
  ddP_ij = d u32 sum_c |dO_ic V_jc|
  eS_ij  = (eP_ij + 2^-8) P_ij |dP_ij - D_i| + P_ij (ddP_ij + dD_i)    (dS, bf16 included)
  |d dV_jc| <= sum_i (eP_ij + 2^-8) P_ij |dO_ic| + Nq u32 sum_i P_ij |dO_ic| + 2^-8 |dV_jc|
  |d dQ_ic| <= scale (sum_j eS_ij |K_jc| + Nk u32 sum_j |dS_ij K_jc|) + 2^-8 |dQ_ic|
  |d dK_jc| <= scale (sum_i eS_ij |Q_ic| + Nq u32 sum_i |dS_ij Q_ic|) + 2^-8 |dK_jc|
each times 1.05 (second-order terms) plus 1e-6.  |dLSE| and |O' - O| are the GPU
forward's own errors, measured in the test against the forward oracle.
"""
import numpy as np
import pytest

import oracle
from io_aware_exact_24_b200.inputs import TENSOR_DO, bf16_bits_to_f32, normal_bf16

from fa_testutil import compare, to_device_bf16, to_host_f64

pytestmark = pytest.mark.gpu

U32 = 2.0 ** -23


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from io_aware_exact_24_b200.build import build
    build()


def run_fwd_bwd(q, k, v, do, scale, causal=False, key_lens=None):
    """fa_fwd then fa_bwd on the GPU.  Returns (O, LSE, dQ, dK, dV) as fp64 numpy."""
    import torch
    from io_aware_exact_24_b200 import fa_bwd, fa_bwd_workspace_size, fa_fwd
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    tq, tk, tv, tdo = (to_device_bf16(x) for x in (q, k, v, do))
    tkl = None if key_lens is None else torch.from_numpy(np.asarray(key_lens, np.int32)).cuda()
    o = torch.empty((B, H, Nq, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device="cuda")
    if Nq > 0:
        fa_fwd(tq, tk if Nk else None, tv if Nk else None, o, lse, B, H, Nq, Nk, d, scale, causal, tkl)
    dq = torch.full((B, H, Nq, d), 3.0, dtype=torch.bfloat16, device="cuda")
    dk = torch.full((B, H, Nk, d), 3.0, dtype=torch.bfloat16, device="cuda")
    dv = torch.full((B, H, Nk, d), 3.0, dtype=torch.bfloat16, device="cuda")
    nbytes = fa_bwd_workspace_size(B, H, Nq, d)
    ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device="cuda")
    fa_bwd(tq if Nq else None, tk if Nk else None, tv if Nk else None, o if Nq else None,
           lse if Nq else None, tdo if Nq else None, dq if Nq else None, dk if Nk else None,
           dv if Nk else None, B, H, Nq, Nk, d, scale, causal, tkl, ws, nbytes)
    torch.cuda.synchronize()
    return (to_host_f64(o), lse.cpu().numpy().astype(np.float64), to_host_f64(dq), to_host_f64(dk),
            to_host_f64(dv))


def bounds(q, k, v, do, scale, causal, kl, o_gpu, lse_gpu):
    """Per-element bounds of the derivation above; returns (ref dQ, dK, dV, bounds)."""
    dq, dk, dv, parts = oracle.attn_bwd_ref(q, k, v, do, scale, causal, kl, return_parts=True)
    o_ref, lse_ref = oracle.attn_ref(q, k, v, scale, causal, kl)
    qf, kf, vf, dof = (bf16_bits_to_f32(x).astype(np.float64) for x in (q, k, v, do))
    B, H, Nq, d = qf.shape
    sc = float(np.float32(scale))
    bq, bk, bv = np.zeros_like(dq), np.zeros_like(dk), np.zeros_like(dv)
    n = 0
    for b in range(B):
        for h in range(H):
            P, dP, D = parts["P"][n], parts["dP"][n], parts["D"][n][:, None]
            n += 1
            fin = np.isfinite(lse_ref[b, h])
            dl = np.where(fin, np.abs(np.where(fin, lse_gpu[b, h], 0) - np.where(fin, lse_ref[b, h], 0)), 0)
            eP = dl[:, None] + d * U32 * sc * (np.abs(qf[b, h]) @ np.abs(kf[b, h]).T) + 2.0 ** -20
            dD = (np.abs(dof[b, h]) * np.abs(o_gpu[b, h] - o_ref[b, h])).sum(1, keepdims=True) + \
                d * U32 * (np.abs(dof[b, h] * o_ref[b, h])).sum(1, keepdims=True)
            ddP = d * U32 * (np.abs(dof[b, h]) @ np.abs(vf[b, h]).T)
            dS = P * (dP - D)
            eS = (eP + 2.0 ** -8) * P * np.abs(dP - D) + P * (ddP + dD)
            Nk = kf.shape[2]
            bv[b, h] = ((eP + 2.0 ** -8) * P).T @ np.abs(dof[b, h]) + Nq * U32 * (P.T @ np.abs(dof[b, h])) + \
                2.0 ** -8 * np.abs(dv[b, h])
            bq[b, h] = sc * (eS @ np.abs(kf[b, h]) + Nk * U32 * (np.abs(dS) @ np.abs(kf[b, h]))) + \
                2.0 ** -8 * np.abs(dq[b, h])
            bk[b, h] = sc * (eS.T @ np.abs(qf[b, h]) + Nq * U32 * (np.abs(dS).T @ np.abs(qf[b, h]))) + \
                2.0 ** -8 * np.abs(dk[b, h])
    f = lambda x: 1.05 * x + 1e-6
    return dq, dk, dv, f(bq), f(bk), f(bv), o_ref, lse_ref


CASES = [
    # B, H, Nq, Nk, d, causal, key_lens
    (1, 2, 1000, 1000, 128, True, None),       # 8 query tiles, ragged tails
    (2, 2, 384, 640, 64, False, [640, 300]),   # key padding
    (1, 2, 300, 520, 64, True, None),          # N_q < N_k: bottom-right diagonal
    (1, 2, 520, 300, 128, True, None),         # N_q > N_k: leading rows see nothing
    (2, 2, 256, 256, 64, False, [0, 256]),     # a sequence with no keys
    (1, 1, 129, 131, 128, False, None),        # one row / key past a tile
]


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_bwd_matches_oracle_within_the_derived_bound(case):
    B, H, Nq, Nk, d, causal, kl = case
    seed = 1300 + Nq + Nk + d
    q = normal_bf16((B, H, Nq, d), seed, 0)
    k = normal_bf16((B, H, Nk, d), seed, 1)
    v = normal_bf16((B, H, Nk, d), seed, 2)
    do = normal_bf16((B, H, Nq, d), seed, TENSOR_DO)
    scale = float(np.float32(1 / np.sqrt(d)))
    kl_arr = None if kl is None else np.array(kl, np.int32)
    o, lse, gq, gk, gv = run_fwd_bwd(q, k, v, do, scale, causal, kl_arr)
    rq, rk, rv, bq, bk, bv, o_ref, lse_ref = bounds(q, k, v, do, scale, causal, kl_arr, o, lse)
    compare(o, lse, o_ref, lse_ref, f"{case} forward")
    worst = {}
    for name, g, r, bd in (("dQ", gq, rq, bq), ("dK", gk, rk, bk), ("dV", gv, rv, bv)):
        assert not np.isnan(g).any(), f"{case}: NaN in {name}"
        ratio = float((np.abs(g - r) / bd).max()) if g.size else 0.0
        rel = float(np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-30))
        worst[name] = (round(ratio, 3), f"{rel:.2e}")
        assert ratio <= 1.0, f"{case}: {name} exceeds its derived bound by x{ratio:.3f} (rel {rel:.2e})"
    print(f"{case}: max |err|/bound and rel Frobenius {worst}")


def test_bwd_keys_no_query_sees_and_queries_without_keys_get_zero():
    # N_q > N_k causal: rows 0..N_q-N_k-1 see nothing (dQ = 0); padding: keys >= key_len
    B, H, Nq, Nk, d = 2, 1, 300, 200, 64
    q, k, v = (normal_bf16((B, H, n, d), 77, t) for n, t in ((Nq, 0), (Nk, 1), (Nk, 2)))
    do = normal_bf16((B, H, Nq, d), 77, TENSOR_DO)
    o, lse, gq, gk, gv = run_fwd_bwd(q, k, v, do, 0.125, True, np.array([200, 50], np.int32))
    assert np.all(gq[:, :, :Nq - Nk] == 0)
    assert np.all(gk[1, :, 50:] == 0) and np.all(gv[1, :, 50:] == 0)


def test_bwd_empty_sides():
    d = 64
    q = normal_bf16((1, 2, 0, d), 5, 0)
    k = normal_bf16((1, 2, 150, d), 5, 1)
    v = normal_bf16((1, 2, 150, d), 5, 2)
    do = normal_bf16((1, 2, 0, d), 5, TENSOR_DO)
    _, _, _, gk, gv = run_fwd_bwd(q, k, v, do, 0.125, False)
    assert np.all(gk == 0) and np.all(gv == 0)          # N_q = 0: no gradient reaches K, V
    q = normal_bf16((1, 2, 140, d), 6, 0)
    k0 = normal_bf16((1, 2, 0, d), 6, 1)
    do = normal_bf16((1, 2, 140, d), 6, TENSOR_DO)
    _, lse, gq, _, _ = run_fwd_bwd(q, k0, k0, do, 0.125, False)
    assert np.all(np.isneginf(lse)) and np.all(gq == 0)  # N_k = 0: dQ = 0


def test_bwd_key_side_is_deterministic():
    B, H, Nq, Nk, d = 1, 2, 700, 600, 128
    q, k, v = (normal_bf16((B, H, n, d), 78, t) for n, t in ((Nq, 0), (Nk, 1), (Nk, 2)))
    do = normal_bf16((B, H, Nq, d), 78, TENSOR_DO)
    a = run_fwd_bwd(q, k, v, do, 0.088, True)
    b = run_fwd_bwd(q, k, v, do, 0.088, True)
    assert np.array_equal(a[3], b[3]) and np.array_equal(a[4], b[4])
    np.testing.assert_allclose(a[2], b[2], rtol=0, atol=1e-2 * np.abs(a[2]).max())
