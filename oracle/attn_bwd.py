"""fp64 CPU oracle for the attention BACKWARD pass -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may
import this module; the product never does.

What it computes: the gradients of the forward's plain definition (attn_ref.c) with
respect to Q, K and V, given the upstream gradient dO of O.  The pages name the step
but print no formula: training needs the backward pass and its recomputation of the
attention matrix ("FlashAttention：把注意力从公式写成数据流", section
"用实验验证而不是背诵结论"; "[2205.14135] FlashAttention: Fast and Memory-Efficient
Exact Attention with IO-Awareness", section "三、FLOPs（計算能力）並非 Speedup 的主因素",
on the extra recomputation FLOPs).  The oracle is the chain rule of that definition,
written out per (b, h) with every matrix materialised:

    S  = scale * Q K^T, masked entries -inf        P  = softmax(S) row-wise
    O  = P V                                        dV = P^T dO
    dP = dO V^T                                     dS = P * (dP - rowsum(dP * P))
    dQ = scale * dS K                               dK = scale * dS^T Q

(rowsum(dP * P)_i = dO_i . O_i.)  Rows with no visible key have P = 0 and contribute
nothing.  Inputs are bf16 bit patterns widened exactly to fp64; outputs are fp64.
Masks follow the forward: key j visible to query i iff j < key_len[b] and, when
causal, j <= i + (N_k - N_q).
"""
from __future__ import annotations

import numpy as np


def _widen(bits):
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def _visible(Nq, Nk, causal, kl):
    i = np.arange(Nq)[:, None]
    j = np.arange(Nk)[None, :]
    vis = np.broadcast_to(j < kl, (Nq, Nk))
    if causal:
        vis = vis & (j <= i + (Nk - Nq))
    return np.ascontiguousarray(vis)


def attn_bwd_ref(q, k, v, do, scale, causal=False, key_lens=None, return_parts=False):
    """Gradients of the plain attention definition.  q [B,H,Nq,d], k/v [B,H,Nk,d],
    do [B,H,Nq,d] bf16 bits; scale the fp32 value the forward uses.
    Returns (dQ, dK, dV) in fp64 (and, with return_parts, a dict of the per-(b,h)
    P, dP, D = rowsum(dP*P) and O lists, for tolerance derivations)."""
    qf, kf, vf, dof = _widen(q), _widen(k), _widen(v), _widen(do)
    B, H, Nq, d = qf.shape
    Nk = kf.shape[2]
    sc = float(np.float32(scale))
    dq = np.zeros_like(qf)
    dk = np.zeros_like(kf)
    dv = np.zeros_like(vf)
    parts = {"P": [], "dP": [], "D": [], "O": []} if return_parts else None
    for b in range(B):
        kl = Nk if key_lens is None else int(min(max(int(key_lens[b]), 0), Nk))
        vis = _visible(Nq, Nk, causal, kl)
        has = vis.any(axis=1)
        for h in range(H):
            S = np.where(vis, sc * (qf[b, h] @ kf[b, h].T), -np.inf)
            m = np.where(has, S.max(axis=1), 0.0)[:, None]
            E = np.where(vis, np.exp(S - m), 0.0)
            l = E.sum(axis=1, keepdims=True)
            P = np.where(has[:, None], E / np.where(l > 0, l, 1.0), 0.0)
            O = P @ vf[b, h]
            dv[b, h] = P.T @ dof[b, h]
            dP = dof[b, h] @ vf[b, h].T
            D = (dP * P).sum(axis=1, keepdims=True)
            dS = P * (dP - D)
            dq[b, h] = sc * (dS @ kf[b, h])
            dk[b, h] = sc * (dS.T @ qf[b, h])
            if return_parts:
                parts["P"].append(P)
                parts["dP"].append(dP)
                parts["D"].append(D[:, 0])
                parts["O"].append(O)
    if return_parts:
        return dq, dk, dv, parts
    return dq, dk, dv
