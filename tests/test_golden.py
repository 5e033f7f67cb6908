"""Hand-worked cases (tests/golden/tiny_cases.json) against both CPU formulations."""
import json
import os

import numpy as np
import pytest

import oracle
from io_aware_exact_24_b200.inputs import bf16_bits_to_f32, f32_to_bf16_bits

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "tiny_cases.json")
with open(GOLDEN) as fh:
    CASES = json.load(fh)["cases"]


def _arr(x, shape):
    a = np.asarray(x, np.float32).reshape(shape)
    bits = f32_to_bf16_bits(a)
    assert np.array_equal(bf16_bits_to_f32(bits), a), "golden input not exact in bf16"
    return bits


def _load(case):
    B, H, Nq, Nk, d = (case[n] for n in ("B", "H", "Nq", "Nk", "d"))
    q = _arr(case["q"], (B, H, Nq, d))
    k = _arr(case["k"], (B, H, Nk, d))
    v = _arr(case["v"], (B, H, Nk, d))
    kl = None if case["key_lens"] is None else np.asarray(case["key_lens"], np.int32)
    o = np.asarray(case["o"], np.float64).reshape(B, H, Nq, d)
    lse = np.asarray([float(x) for x in case["lse"]], np.float64).reshape(B, H, Nq)
    return q, k, v, kl, o, lse


@pytest.mark.parametrize("case", CASES, ids=[c["name"] for c in CASES])
@pytest.mark.parametrize("which", ["ref", "online"])
def test_golden_case(case, which):
    q, k, v, kl, o_exp, lse_exp = _load(case)
    fn = oracle.attn_ref if which == "ref" else oracle.attn_online
    o, lse = fn(q, k, v, case["scale"], case["causal"], kl)
    np.testing.assert_allclose(o, o_exp, rtol=0, atol=1e-15)
    assert np.array_equal(np.isneginf(lse), np.isneginf(lse_exp))
    fin = np.isfinite(lse_exp)
    np.testing.assert_allclose(lse[fin], lse_exp[fin], rtol=0, atol=1e-15)
