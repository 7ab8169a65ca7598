"""Pins of the oracle's FP8 linear layer (gemm_e4m3) against what the definition fixes: a
brute-force triple loop on a tiny case, a constant-code case with a closed form, and exact
linearity in each scale (powers of two)."""
import numpy as np

import oracle


def _codes(rng, shape):
    c = rng.integers(0, 256, size=shape, dtype=np.uint8)
    c[(c & 0x7F) == 0x7F] = 0x38               # no NaN codes
    return c


def test_gemm_matches_a_triple_loop():
    rng = np.random.default_rng(5)
    a8, b8 = _codes(rng, (3, 5)), _codes(rng, (4, 5))
    y, bound = oracle.gemm_e4m3(a8, b8, 0.5, 0.25)
    for m in range(3):
        for n in range(4):
            want = sum(oracle.e4m3_to_float(int(a8[m, k])) * 0.5 *
                       oracle.e4m3_to_float(int(b8[n, k])) * 0.25 for k in range(5))
            mag = sum(abs(oracle.e4m3_to_float(int(a8[m, k])) * 0.5 *
                          oracle.e4m3_to_float(int(b8[n, k])) * 0.25) for k in range(5))
            assert y[m, n] == want and bound[m, n] == mag


def test_gemm_constant_codes_closed_form():
    # code 0x38 is 1.0, code 0x40 is 2.0: every output is K * 1 * 2 * s_a * s_b
    K = 384
    y, _ = oracle.gemm_e4m3(np.full((7, K), 0x38, np.uint8), np.full((9, K), 0x40, np.uint8), 3.0, 0.125)
    assert np.all(y == K * 2.0 * 3.0 * 0.125)


def test_gemm_is_linear_in_each_scale_and_rows_select():
    rng = np.random.default_rng(6)
    a8, b8 = _codes(rng, (6, 256)), _codes(rng, (32, 256))
    y1, _ = oracle.gemm_e4m3(a8, b8, 1.0, 1.0)
    y2, _ = oracle.gemm_e4m3(a8, b8, 4.0, 0.5)
    assert np.array_equal(y2, 2.0 * y1)        # powers of two: exact in FP64
    y3, _ = oracle.gemm_e4m3(a8, b8, 1.0, 1.0, rows=[4, 1])
    assert np.array_equal(y3, y1[[4, 1]])
