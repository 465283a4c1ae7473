"""Pins of the oracle's fused_qk_norm_rope against independent routines,
closed forms and the invariants of a rotation."""
import numpy as np
import pytest

import fp8q_inputs as inp
import oracle

HQ, HK, HV, D = 4, 2, 2, 128


def _cache(P, D, seed):
    # rope cache as a model builds it: theta_i = base^(-2i/D), angle = p * theta_i
    inv = 1.0 / (1e6 ** (np.arange(0, D, 2) / D))
    ang = np.arange(P)[:, None] * inv[None, :]
    return np.concatenate([np.cos(ang), np.sin(ang)], axis=1).astype(np.float32)


def _inputs(T, seed):
    qkv = inp.to_bf16_bits(np.random.default_rng(seed).uniform(-0.1, 0.1, size=(T, (HQ + HK + HV) * D)))
    return qkv, inp.rms_weight_bf16(seed + 1, D), inp.rms_weight_bf16(seed + 2, D)


def _head_norm(qkv, h, w):
    """Per-head RMSNorm values through the oracle's RMSNorm quant (an independent path)."""
    rows = qkv[:, h * D:(h + 1) * D]
    _, _, y = oracle.rmsnorm_quant(rows, w, 1e-6, D, want_y=True)
    return y.astype(np.float64)


@pytest.mark.parametrize("neox", [True, False])
def test_position_zero_is_the_per_head_rmsnorm(neox):
    # cos = 1, sin = 0 at position 0: the op reduces to RMSNorm of every q/k head
    qkv, qw, kw = _inputs(5, 1)
    cs = _cache(4, D, 0)
    out = oracle.qk_norm_rope(qkv, HQ, HK, HV, D, 1e-6, qw, kw, cs, np.zeros(5, np.int64), neox)
    for h in range(HQ + HK):
        y = _head_norm(qkv, h, qw if h < HQ else kw)
        np.testing.assert_array_equal(inp.bf16_bits_to_f32(out[:, h * D:(h + 1) * D]), y.astype(np.float32))
    np.testing.assert_array_equal(out[:, (HQ + HK) * D:], qkv[:, (HQ + HK) * D:])    # v untouched


@pytest.mark.parametrize("neox", [True, False])
def test_quarter_turn_is_a_signed_permutation(neox):
    # cos = 0, sin = 1: out_a = -y_b, out_b = y_a exactly
    qkv, qw, kw = _inputs(3, 2)
    cs = np.concatenate([np.zeros((1, D // 2)), np.ones((1, D // 2))], axis=1).astype(np.float32)
    out = oracle.qk_norm_rope(qkv, HQ, HK, HV, D, 1e-6, qw, kw, cs, np.zeros(3, np.int64), neox)
    for h in range(HQ + HK):
        y = _head_norm(qkv, h, qw if h < HQ else kw)
        o = inp.bf16_bits_to_f32(out[:, h * D:(h + 1) * D]).astype(np.float64)
        a = np.arange(D // 2) if neox else 2 * np.arange(D // 2)
        b = a + D // 2 if neox else a + 1
        np.testing.assert_array_equal(o[:, a], -y[:, b])
        np.testing.assert_array_equal(o[:, b], y[:, a])


def test_rotation_keeps_pair_norms():
    # |out_a|^2 + |out_b|^2 = |y_a|^2 + |y_b|^2 up to the two bf16 roundings
    qkv, qw, kw = _inputs(6, 3)
    cs = _cache(1000, D, 0)
    pos = np.array([0, 1, 17, 500, 999, 3], np.int64)
    out = oracle.qk_norm_rope(qkv, HQ, HK, HV, D, 1e-6, qw, kw, cs, pos, True)
    for h in range(HQ + HK):
        y = _head_norm(qkv, h, qw if h < HQ else kw)
        o = inp.bf16_bits_to_f32(out[:, h * D:(h + 1) * D]).astype(np.float64)
        ny = y[:, :D // 2] ** 2 + y[:, D // 2:] ** 2
        no = o[:, :D // 2] ** 2 + o[:, D // 2:] ** 2
        assert np.all(np.abs(no - ny) <= 2 * 2.0 ** -8 * ny + 1e-30)


def test_gptj_is_neox_on_interleaved_dims():
    # permuting the head dims (pairs (2i, 2i+1) <-> (i, i + D/2)) maps one style onto the
    # other; RMSNorm is equivariant when the weight is permuted the same way
    qkv, qw, kw = _inputs(4, 4)
    cs = _cache(64, D, 0)
    pos = np.array([3, 9, 0, 63], np.int64)
    perm = np.empty(D, np.int64)
    perm[0::2] = np.arange(D // 2)
    perm[1::2] = np.arange(D // 2) + D // 2          # gptj position j holds neox dim perm[j]
    cols = np.concatenate([h * D + perm for h in range(HQ + HK + HV)])
    neox = oracle.qk_norm_rope(qkv, HQ, HK, HV, D, 1e-6, qw, kw, cs, pos, True)
    gptj = oracle.qk_norm_rope(qkv[:, cols], HQ, HK, HV, D, 1e-6, qw[perm], kw[perm], cs, pos, False)
    np.testing.assert_array_equal(gptj, neox[:, cols])


def test_hand_case_small_head():
    # D = 4, one q head: x = (3, 4, 0, 0) -> mean(x^2) = 25/4, r = 2/5 (eps 0): n = (1.2, 1.6, 0, 0)
    # rounded to bf16, w = 1; position 0 of a cache with angle pi/2 on pair 0, 0 on pair 1:
    # neox pairs (0, 2), (1, 3): out0 = -y2 = 0, out2 = y0, out1 = y1 (cos 1), out3 = y3 = 0
    x = inp.to_bf16_bits(np.array([[3.0, 4.0, 0.0, 0.0]]))
    one = inp.to_bf16_bits(np.ones(4))
    cs = np.array([[0.0, 1.0, 1.0, 0.0]], np.float32)          # cos (pair0, pair1), sin (pair0, pair1)
    out = oracle.qk_norm_rope(x, 1, 0, 0, 4, 0.0, one, one, cs, np.zeros(1, np.int64), True)
    b12 = float(inp.bf16_bits_to_f32(inp.to_bf16_bits(np.array([1.2])))[0])
    b16 = float(inp.bf16_bits_to_f32(inp.to_bf16_bits(np.array([1.6])))[0])
    np.testing.assert_array_equal(inp.bf16_bits_to_f32(out[0]), np.array([0.0, b16, b12, 0.0], np.float32))
