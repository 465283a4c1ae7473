"""Pins of the oracle's W8A8_INT8 functions (int8 codes, scale amax/127,
exact integer GEMM) against independent routines, closed forms and invariants."""
import numpy as np
import pytest

import fp8q_inputs as inp
import oracle


def test_int8_encode_is_numpy_rint_saturated():
    # numpy's rint rounds half to even; every fp32 pattern between -140 and 140
    # on a dense grid (quarter and half-integer ties included), plus extremes
    g = np.random.default_rng(1)
    v = np.concatenate([np.arange(-140, 140, 0.25), g.uniform(-200, 200, 200000),
                        [0.5, 1.5, 2.5, -0.5, -2.5, 126.5, 127.49, 127.5, -128.5, -129.0, 1e30, -1e30,
                         np.nextafter(np.float32(0.5), np.float32(1)), 0.0, -0.0]]).astype(np.float32)
    q, _ = oracle.int8_quantize(np.ones((1, 1), np.float32), 1)   # warm the library
    got = np.array([oracle.int8_encode_scalar(float(t)) for t in v[:2000]], np.int8)
    want = np.clip(np.rint(v[:2000].astype(np.float64)), -128, 127).astype(np.int8)
    np.testing.assert_array_equal(got, want)
    np.testing.assert_array_equal(
        np.array([oracle.int8_encode_scalar(float(t)) for t in v[-15:]], np.int8),
        np.clip(np.rint(v[-15:].astype(np.float64)), -128, 127).astype(np.int8))
    # the array path: codes of fl32(y / s) for a row of the random values
    y = v[2000:-15].reshape(1, -1)
    q, s = oracle.int8_quantize(y, y.shape[1])
    ratio = (y[0] / s[0, 0]).astype(np.float32)
    np.testing.assert_array_equal(q[0], np.clip(np.rint(ratio.astype(np.float64)), -128, 127).astype(np.int8))
    assert np.abs(q[0].astype(np.int32)).max() == 127


def test_int8_scale_hand_cases():
    assert oracle._load().oracle_int8_scale(127.0) == 1.0
    assert oracle._load().oracle_int8_scale(0.0) == np.float32(np.float32(1e-10) / np.float32(127.0))
    assert oracle._load().oracle_int8_scale(1.0) == np.float32(1.0) / np.float32(127.0)


@pytest.mark.parametrize("g", [128, 512])
def test_int8_quant_invariants(g):
    # the amax element maps to exactly +-127; |q*s - y| <= s/2 (+ the fp32 rounding
    # of y/s); an all-zero group takes the floored scale and zero codes
    y = inp.bf16_bits_to_f32(inp.heavy_tailed_bf16(5, 6, 512)).reshape(6, 512).copy()
    y[2, :128] = 0.0
    q, s = oracle.int8_quantize(y, g)
    G = 512 // g
    for m in range(6):
        for j in range(G):
            v = y[m, j * g:(j + 1) * g].astype(np.float64)
            c = q[m, j * g:(j + 1) * g].astype(np.float64)
            sc = float(s[m, j])
            amax = np.abs(v).max()
            if amax == 0:
                assert sc == np.float32(np.float32(1e-10) / np.float32(127.0)) and np.all(c == 0)
                continue
            assert np.abs(c[np.argmax(np.abs(v))]) == 127
            assert np.all(np.abs(c * sc - v) <= 0.5 * sc * (1 + 1e-6) + 1e-30)


def test_int8_producers_share_the_fp8_readings():
    # the int8 producer ops quantize exactly the values the fp8 ops quantize
    x = inp.heavy_tailed_bf16(6, 4, 1024)
    w = inp.rms_weight_bf16(7, 1024)
    _, _, y = oracle.rmsnorm_quant(x, w, 1e-6, 128, want_y=True)
    q, s = oracle.rmsnorm_quant_i8(x, w, 1e-6, 128)
    q2, s2 = oracle.int8_quantize(y, 128)
    np.testing.assert_array_equal(q, q2)
    np.testing.assert_array_equal(s, s2)
    xs = inp.normal_bf16(8, (3, 512), std=3.0)
    _, _, ys = oracle.silu_mul_quant(xs, 256, want_y=True)
    np.testing.assert_array_equal(oracle.silu_mul_quant_i8(xs, 256)[0], oracle.int8_quantize(ys, 256)[0])


@pytest.mark.parametrize("per_token,per_channel", [(True, True), (False, True), (True, False)])
def test_scaled_mm_i8_brute_force(per_token, per_channel):
    # Python integers and fractions: exact dot products, fp64 scaling
    from fractions import Fraction
    g = np.random.default_rng(9)
    M, N, K = 5, 7, 96
    a = g.integers(-128, 128, size=(M, K)).astype(np.int8)
    b = g.integers(-128, 128, size=(N, K)).astype(np.int8)
    sa = inp.random_scales(10, (M if per_token else 1,))
    sb = inp.random_scales(11, (N if per_channel else 1,))
    y, ad = oracle.scaled_mm_i8(a, b, sa, sb)
    for m in range(M):
        for n in range(N):
            dot = sum(int(a[m, k]) * int(b[n, k]) for k in range(K))
            sc = Fraction(float(sa[m if per_token else 0])) * Fraction(float(sb[n if per_channel else 0]))
            assert abs(Fraction(y[m, n]) - dot * sc) <= abs(dot * sc) * Fraction(1, 2 ** 52)
            absdot = sum(abs(int(a[m, k]) * int(b[n, k])) for k in range(K))
            assert abs(Fraction(ad[m, n]) - absdot * abs(sc)) <= absdot * abs(sc) * Fraction(1, 2 ** 52)


def test_scaled_mm_i8_rows_and_transposition():
    # a non-square identity-like B catches a transposed operand; row selection
    M, K = 4, 64
    a = np.random.default_rng(12).integers(-100, 100, size=(M, K)).astype(np.int8)
    b = np.zeros((K, K), np.int8)
    b[np.arange(K), np.arange(K)] = 1
    y, _ = oracle.scaled_mm_i8(a, b, np.ones(M, np.float32), np.ones(K, np.float32))
    np.testing.assert_array_equal(y, a.astype(np.float64))
    y2, _ = oracle.scaled_mm_i8(a, b, np.ones(M, np.float32), np.ones(K, np.float32), rows=np.array([3, 1]))
    np.testing.assert_array_equal(y2, a[[3, 1]].astype(np.float64))
