"""CPU checks of the derived parity bounds used by the E4M3 and backward GPU tests.

Each test emulates, in numpy, the roundings the kernel performs (E4M3 probabilities
normalised by their rounded sum; bf16 P and dS with fp32 sums for the backward) and
checks that a correct implementation of that arithmetic stays inside the bound the GPU
test applies -- i.e. that the bound is not tighter than the arithmetic allows -- and
that a plausible mistake (normalising by the unrounded sum, dropping D) breaks it.
"""
import numpy as np
import pytest

import oracle
from io_aware_exact_24_b200.inputs import TENSOR_DO, bf16_bits_to_f32, f32_to_bf16_bits, normal_bf16

torch = pytest.importorskip("torch")

from test_gpu_bwd import bounds  # noqa: E402
from test_gpu_fp8 import _inputs, _visible, bound_rows  # noqa: E402


def _bf(x):
    return bf16_bits_to_f32(f32_to_bf16_bits(np.asarray(x, np.float32))).astype(np.float64)


def _e4m3(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.float8_e4m3fn).to(torch.float64).numpy()


def _fp8_case():
    B, H, Nq, Nk = 1, 1, 300, 400
    q8, k8, v8, qd, kd, vd = _inputs(B, H, Nq, Nk, 5)
    scale = float(np.float32(1 / np.sqrt(128)))
    o_ref, _ = oracle.attn_ref_e4m3(q8, k8, v8, scale, qd, kd, vd, True)
    s_eff = float(np.float32(np.float64(scale) * qd * kd))
    qf, kf = oracle.e4m3_to_f64(q8[0, 0]), oracle.e4m3_to_f64(k8[0, 0])
    vf = oracle.e4m3_to_f64(v8[0, 0]) * np.float64(np.float32(vd))
    vis = _visible(Nq, Nk, True, Nk)
    S = np.where(vis, (qf @ kf.T) * s_eff, -np.inf)
    e = np.exp(S - S.max(axis=1, keepdims=True))
    return o_ref[0, 0], qf, kf, vf, s_eff, vis, e, float(np.float32(vd))


@pytest.mark.parametrize("F", [1.0, 37.0, 255.0])
def test_e4m3_bound_holds_for_the_rounded_probabilities(F):
    o_ref, qf, kf, vf, s_eff, vis, e, _ = _fp8_case()
    p = _e4m3(e * F)                                   # the kernel's p, up to 2^8 above e
    o = _bf((p @ vf) / p.sum(axis=1, keepdims=True))   # O normalised by the rounded sum
    bd = bound_rows(qf, kf, vf, s_eff, vis, o_ref)
    assert (np.abs(o - o_ref) / bd).max() <= 1.0


def test_e4m3_bound_catches_a_dropped_v_descale():
    # The bound is a worst-case (triangle-inequality) bound: on random rows it still
    # admits rounding P even more coarsely, so it guards against wrong results, not
    # against a last bit of precision.  A plumbing slip is far outside it.
    o_ref, qf, kf, vf, s_eff, vis, e, vd = _fp8_case()
    p = _e4m3(e)
    o = _bf((p @ (vf / vd)) / p.sum(axis=1, keepdims=True))   # V descale left out
    bd = bound_rows(qf, kf, vf, s_eff, vis, o_ref)
    assert (np.abs(o - o_ref) / bd).max() > 1.0


def _bwd_case(drop_d=False):
    B, H, N, d = 1, 1, 400, 64
    q, k, v, do = (normal_bf16((B, H, N, d), 21, t) for t in (0, 1, 2, TENSOR_DO))
    scale = float(np.float32(1 / np.sqrt(d)))
    o_ref, lse_ref = oracle.attn_ref(q, k, v, scale, True)
    o_g, lse_g = _bf(o_ref), lse_ref.astype(np.float32).astype(np.float64)
    rq, rk, rv, bq, bk, bv, _, _ = bounds(q, k, v, do, scale, True, None, o_g, lse_g)
    qf, kf, vf, dof = (bf16_bits_to_f32(x)[0, 0] for x in (q, k, v, do))
    c = np.float32(scale * 1.4426950408889634)
    S = (qf @ kf.T).astype(np.float32)
    vis = np.tril(np.ones((N, N), bool))
    l2 = (lse_g[0, 0] * 1.4426950408889634).astype(np.float32)[:, None]
    P = np.where(vis, np.exp2(S * c - l2), 0).astype(np.float32)
    D = (dof * o_g[0, 0].astype(np.float32)).sum(axis=1).astype(np.float32)
    dP = (dof @ vf.T).astype(np.float32)
    dS = P * (dP - (0 if drop_d else D[:, None]))
    Pb, dSb = _bf(P), _bf(dS)
    got = (_bf(scale * (dSb @ kf)), _bf(scale * (dSb.T @ qf)), _bf(Pb.T @ dof))
    ref = (rq[0, 0], rk[0, 0], rv[0, 0])
    bd = (bq[0, 0], bk[0, 0], bv[0, 0])
    return [float((np.abs(g - r) / b).max()) for g, r, b in zip(got, ref, bd)]


def test_backward_bounds_hold_for_bf16_p_and_ds():
    assert max(_bwd_case()) <= 1.0


def test_backward_bounds_catch_a_dropped_d_term():
    rq, rk, rv = _bwd_case(drop_d=True)
    assert rq > 1.0 and rk > 1.0
