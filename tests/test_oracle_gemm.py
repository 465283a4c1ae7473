"""Pins of the oracle's scaled FP8 GEMMs.

Brute force with exact rationals (``oracle.exact``, which decodes codes with
ml_dtypes) on tiny shapes, closed forms with identity-like weights, and the
agreement of the blockwise GEMM with the per-channel one when every block of a
row carries the same scale.
"""
import numpy as np
import pytest

import fp8q_inputs as inp
import oracle
from oracle import exact


def _close_to_exact(y, ad, ex):
    ex = np.array([[float(v) for v in row] for row in ex])
    assert np.all(np.abs(y - ex) <= 1e-13 * ad + 1e-300), np.abs(y - ex).max()


@pytest.mark.parametrize("M,N,K", [(1, 1, 16), (3, 5, 32), (7, 4, 48)])
@pytest.mark.parametrize("per_token,per_channel", [(True, True), (False, True), (True, False)])
def test_scaled_mm_exact_rationals(M, N, K, per_token, per_channel):
    a = inp.random_e4m3_codes(M * 100 + N, (M, K))
    b = inp.random_e4m3_codes(K * 10 + 1, (N, K))
    sa = inp.random_scales(1, (M if per_token else 1,))
    sb = inp.random_scales(2, (N if per_channel else 1,))
    y, ad = oracle.scaled_mm(a, b, sa, sb)
    _close_to_exact(y, ad, exact.scaled_mm_exact(a, b, sa, sb))


@pytest.mark.parametrize("M,N,K", [(2, 128, 256), (3, 256, 128)])
def test_scaled_mm_blockwise_exact_rationals(M, N, K):
    a = inp.random_e4m3_codes(M + N + K, (M, K))
    b = inp.random_e4m3_codes(N * 3 + K, (N, K))
    sa = inp.random_scales(3, (M, K // 128))
    sb = inp.random_scales(4, (N // 128, K // 128))
    y, ad = oracle.scaled_mm_blockwise(a, b, sa, sb)
    _close_to_exact(y, ad, exact.scaled_mm_blockwise_exact(a, b, sa, sb))


def test_scaled_mm_identity_weights():
    # B = 1.0 on the diagonal -> y[m, n] = dequant(a[m, n]) * sa[m] * sb[n]; non-square
    # A (M != K) catches a transposed operand.
    M, K = 5, 64
    N = K
    a = inp.random_e4m3_codes(9, (M, K))
    b = np.zeros((N, K), np.uint8)
    b[np.arange(N), np.arange(N)] = 0x38                                 # e4m3 1.0
    sa = inp.random_scales(10, (M,))
    sb = inp.random_scales(11, (N,))
    y, _ = oracle.scaled_mm(a, b, sa, sb)
    import ml_dtypes
    deq = a.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    want = deq * sa.astype(np.float64)[:, None] * sb.astype(np.float64)[None, :]
    np.testing.assert_array_equal(y, want)


def test_blockwise_identity_weights_pick_block_scales():
    M, K, N = 3, 256, 256
    a = inp.random_e4m3_codes(12, (M, K))
    b = np.zeros((N, K), np.uint8)
    b[np.arange(N), np.arange(N)] = 0x38
    sa = inp.random_scales(13, (M, K // 128))
    sb = inp.random_scales(14, (N // 128, K // 128))
    y, _ = oracle.scaled_mm_blockwise(a, b, sa, sb)
    import ml_dtypes
    deq = a.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    n = np.arange(N)
    want = deq * sa.astype(np.float64)[:, n // 128] * sb.astype(np.float64)[n // 128, n // 128]
    np.testing.assert_array_equal(y, want)


def test_blockwise_reduces_to_per_channel():
    # With sa[m, kb] = sa[m] for every kb and sb[nb, kb] = c[nb], blockwise equals
    # scaled_mm with per-token sa and per-channel sb[n] = c[n // 128].
    M, N, K = 4, 256, 384
    a = inp.random_e4m3_codes(15, (M, K))
    b = inp.random_e4m3_codes(16, (N, K))
    sa1 = inp.random_pow2_scales(17, (M,))
    c = inp.random_pow2_scales(18, (N // 128,))
    yb, adb = oracle.scaled_mm_blockwise(a, b, np.repeat(sa1[:, None], K // 128, 1),
                                         np.repeat(c[:, None], K // 128, 1))
    yc, adc = oracle.scaled_mm(a, b, sa1, np.repeat(c, 128))
    assert np.all(np.abs(yb - yc) <= 1e-14 * adc)
    np.testing.assert_allclose(adb, adc, rtol=1e-14)


def test_row_subset_matches_full():
    M, N, K = 9, 40, 64
    a = inp.random_e4m3_codes(19, (M, K))
    b = inp.random_e4m3_codes(20, (N, K))
    sa = inp.random_scales(21, (M,))
    sb = inp.random_scales(22, (N,))
    y, ad = oracle.scaled_mm(a, b, sa, sb)
    rows = np.array([8, 0, 3])
    ys, ads = oracle.scaled_mm(a, b, sa, sb, rows)
    np.testing.assert_array_equal(ys, y[rows])
    np.testing.assert_array_equal(ads, ad[rows])


@pytest.mark.parametrize("M,N,K", [(2, 128, 256), (3, 256, 384)])
def test_scaled_mm_blockwise_e8m0_exact_rationals(M, N, K):
    # E8M0 scale bytes decoded by an independent library (ml_dtypes) into the
    # exact-rational GEMM must agree with the oracle's E8M0 entry.
    import ml_dtypes
    a = inp.random_e4m3_codes(M + 7 * K, (M, K))
    b = inp.random_e4m3_codes(N + 5 * K, (N, K))
    g = np.random.default_rng(M + N)
    sa = g.integers(100, 140, size=(M, K // 128)).astype(np.uint8)
    sb = g.integers(110, 130, size=(N // 128, K // 128)).astype(np.uint8)
    y, ad = oracle.scaled_mm_blockwise_e8m0(a, b, sa, sb)
    dec = lambda t: t.view(ml_dtypes.float8_e8m0fnu).astype(np.float32)
    _close_to_exact(y, ad, exact.scaled_mm_blockwise_exact(a, b, dec(sa), dec(sb)))


def test_gate_up_silu_quant_is_the_chain_on_the_exact_gemm():
    # h = bf16 of the blockwise GEMM, compared with bf16 of the exact-rational
    # GEMM (an independent computation); then the SiLU*mul quant of that h
    M, I, K = 3, 128, 256
    a = inp.random_e4m3_codes(71, (M, K))
    b = inp.random_e4m3_codes(72, (2 * I, K))
    sa = inp.random_scales(73, (M, K // 128))
    sb = inp.random_scales(74, (2 * I // 128, K // 128))
    q, s, h = oracle.gate_up_silu_quant(a, b, sa, sb, 128)
    ex = exact.scaled_mm_blockwise_exact(a, b, sa, sb)
    hx = np.array([[float(v) for v in row] for row in ex])
    # the exact values, rounded to bf16 once by the (separately pinned) bf16 rounding
    want = np.array([[np.float32(oracle.bf16_round(np.array([v]))[0]) for v in row] for row in hx])
    np.testing.assert_array_equal(inp.bf16_bits_to_f32(h), want)
    q2, s2 = oracle.silu_mul_quant(h, 128)
    np.testing.assert_array_equal(q, q2)
    np.testing.assert_array_equal(s, s2)
