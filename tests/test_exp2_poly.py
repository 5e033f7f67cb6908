"""The kernel's FMA-pipe exp2 (range reduction + fitted cubic): constants in sync with
their generator, and the fp32 sequence within its stated relative error everywhere the
kernel uses it (x in [-125, 8])."""
import importlib.util
import os
import re

import numpy as np

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "io_aware_exact_24_b200", "csrc")


def _fit_module():
    spec = importlib.util.spec_from_file_location("exp2_poly_fit",
                                                  os.path.join(CSRC, "exp2_poly_fit.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _header_constants():
    text = open(os.path.join(CSRC, "exp2_poly.cuh")).read()
    return [float(re.search(rf"kExp2C{i} = ([-0-9.e]+)f;", text).group(1)) for i in range(4)]


def test_header_matches_generator():
    fit = _fit_module()
    c, err = fit.remez_relative()
    assert [float(np.float32(v)) for v in c] == _header_constants()
    assert err < 1e-4


def test_emulated_exp2_error_bound():
    fit = _fit_module()
    c = _header_constants()
    xs = np.concatenate([np.linspace(-125, 8, 1_000_001, dtype=np.float32),
                         np.arange(-125, 9, dtype=np.float32),            # integers
                         np.arange(-125, 8, dtype=np.float32) + 0.5,      # ties of the rounding
                         np.float32([-1e-30, 1e-30, -0.0, 0.0])])
    got = fit.emulated_exp2_f32(xs, c).astype(np.float64)
    rel = np.abs(got / np.exp2(xs.astype(np.float64)) - 1)
    assert rel.max() < 1e-4
    # continuity at the reduction boundaries: no jump larger than the error bound
    assert np.all(np.diff(got[:1_000_001]) >= 0)


def test_error_is_far_below_bf16_spacing():
    # probabilities are rounded to bf16 (relative spacing 2^-8) before the PV product
    assert 1e-4 < 2.0 ** -8 / 20
