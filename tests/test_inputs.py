"""Seeded input generator: determinism, bf16 rounding, workload recipe."""
import numpy as np

from io_aware_exact_24_b200.inputs import (WORKLOADS, WORKLOAD_ORDER, bf16_bits_to_f32,
                                           f32_to_bf16_bits, key_lengths, make_inputs,
                                           normal_bf16)


def test_round_to_nearest_even_cases():
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7: rounds to the even mantissa (1.0)
    x = np.array([1.0, 1 + 2**-8, 1 + 3 * 2**-8, 1 + 2**-8 + 2**-20, -2.5, 0.0, -0.0,
                  np.float32(3.4e38)], np.float32)
    got = bf16_bits_to_f32(f32_to_bf16_bits(x))
    exp = np.array([1.0, 1.0, 1 + 4 * 2**-8, 1 + 2**-7, -2.5, 0.0, -0.0, np.inf], np.float32)
    assert np.array_equal(got, exp)
    assert f32_to_bf16_bits(np.float32(-0.0)) == 0x8000


def test_rounding_is_nearest_for_random_values():
    x = np.random.default_rng(0).standard_normal(100000).astype(np.float32)
    r = bf16_bits_to_f32(f32_to_bf16_bits(x)).astype(np.float64)
    err = np.abs(r - x)
    ulp = np.spacing(np.abs(r).astype(np.float32)).astype(np.float64) * 2**16
    assert np.all(err <= ulp / 2 + 1e-30)


def test_generator_is_deterministic_and_streams_differ():
    a = normal_bf16((2, 3, 5, 8), 7, 0)
    b = normal_bf16((2, 3, 5, 8), 7, 0)
    c = normal_bf16((2, 3, 5, 8), 7, 1)
    assert np.array_equal(a, b) and not np.array_equal(a, c)
    half = bf16_bits_to_f32(normal_bf16((4096,), 3, 2, 0.5))
    full = bf16_bits_to_f32(normal_bf16((4096,), 3, 2, 1.0))
    assert np.array_equal(half, full * 0.5)   # sigma 0.5 is an exact power of two


def test_key_lengths_in_range():
    kl = key_lengths(10000, 128, 512, 3)
    assert kl.dtype == np.int32 and kl.min() >= 128 and kl.max() <= 512
    assert kl.min() == 128 and kl.max() == 512   # both ends reachable


def test_workload_shapes():
    assert WORKLOAD_ORDER == list(WORKLOADS)
    x = make_inputs(WORKLOADS["bert_padded_512"])
    assert x["q"].shape == (16, 16, 512, 64) and x["key_lens"].shape == (16,)
    w = WORKLOADS["causal_8000_d128"]
    assert w.flop == 4 * 2 * 32 * 8000 * 8000 * 128 / 2
    assert WORKLOADS["long_16k_d64"].flop == 4 * 16 * 16384**2 * 64


def test_window_flop_counts_visible_pairs():
    from io_aware_exact_24_b200.inputs import Workload
    for Nq, Nk, causal, W in ((9, 9, True, 3), (5, 12, True, 0), (12, 5, True, 2), (6, 10, False, 4)):
        w = Workload("t", 2, 3, Nq, Nk, 8, causal, 0.1, window_left=W)
        pairs = sum(1 for i in range(Nq) for j in range(Nk)
                    if j >= i + Nk - Nq - W and (not causal or j <= i + Nk - Nq))
        assert w.flop == 4.0 * 2 * 3 * 8 * pairs


def test_e4m3_inputs_are_the_bf16_tensors_quantised():
    import oracle
    from io_aware_exact_24_b200.inputs import normal_e4m3

    shape = (2, 3, 70, 64)
    codes, s = normal_e4m3(shape, 4, 1, 0.5)
    x = np.random.Generator(np.random.Philox(key=4 * 16 + 1)).standard_normal(size=shape, dtype=np.float32)
    x = x * np.float32(0.5)
    assert np.float32(s) == np.float32(np.abs(x).max() / 448.0)
    y = oracle.e4m3_to_f64(codes) * s
    # round to nearest: half an ulp, 2^-4 relative for normals, 2^-10 * s absolute below 2^-6 * s
    err = np.abs(y - x.astype(np.float64))
    bound = np.maximum(np.abs(x) * 2.0 ** -4, 2.0 ** -10 * s) * (1 + 1e-6)
    assert np.all(err <= bound)
    assert np.abs(oracle.e4m3_to_f64(codes)).max() == 448.0   # the largest |x| maps to 448
