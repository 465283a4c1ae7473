"""Pins of the oracle's activation-quantization ops.

Invariants fixed by the definition of dynamic quantization (scale =
max(amax,1e-10)/448, q = e4m3(x/scale)): the amax element maps to exactly
+-448, the dequantization error is at most half an e4m3 ULP times the scale,
an all-zero group takes the floored scale; UE8M0 properties; and the
hand-derived closed forms of the RMSNorm and SiLU*mul producers.
"""
import ml_dtypes
import numpy as np
import pytest

import fp8q_inputs as inp
import oracle


def _e4m3_half_ulp(t: np.ndarray) -> np.ndarray:
    a = np.minimum(np.abs(t.astype(np.float64)), 448.0)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -6)))
    return np.ldexp(1.0, (e - 3).astype(int)) / 2


def _dequant(q):
    return q.view(ml_dtypes.float8_e4m3fn).astype(np.float64)


def _cases():
    return [
        ("normal", inp.normal_bf16(1, (33, 512))),
        ("heavy", inp.heavy_tailed_bf16(2, 17, 1024)),
        ("small", inp.normal_bf16(3, (9, 256), std=1e-6)),
    ]


@pytest.mark.parametrize("ue8m0", [False, True])
@pytest.mark.parametrize("per_token", [False, True])
@pytest.mark.parametrize("name,x", _cases())
def test_group_quant_invariants(name, x, per_token, ue8m0):
    M, K = x.shape
    g = K if per_token else 128
    q, s, y = oracle.group_quant(x, g, ue8m0, want_y=True)
    np.testing.assert_array_equal(y, inp.bf16_bits_to_f32(x))        # y is x itself
    yg = y.reshape(M, K // g, g).astype(np.float64)
    qg = _dequant(q).reshape(M, K // g, g)
    amax = np.abs(yg).max(-1)
    sv = s.astype(np.float64)
    # amax element -> exactly +-448 (not in UE8M0 mode, where the scale grew)
    if not ue8m0:
        idx = np.abs(yg).argmax(-1)
        top = np.take_along_axis(qg, idx[..., None], -1)[..., 0]
        nz = amax > 1e-10
        np.testing.assert_array_equal(np.abs(top[nz]), 448.0)
    else:
        assert np.all(np.frexp(sv)[0] == 0.5)
        assert np.abs(qg).max() <= 448.0
    # dequant error <= half an e4m3 ULP of x/s, times s (plus one fp32 rounding of x/s)
    t = (y.reshape(M, K // g, g) / s[..., None]).astype(np.float32)
    err = np.abs(qg * sv[..., None] - yg)
    bound = (_e4m3_half_ulp(t) + np.abs(t) * 2.0 ** -23) * sv[..., None]
    assert np.all(err <= bound)


@pytest.mark.parametrize("ue8m0", [False, True])
def test_all_zero_group_takes_floor_scale(ue8m0):
    x = inp.normal_bf16(4, (3, 384))
    x[1, :] = 0
    x[2, 128:256] = 0
    q, s = oracle.group_quant(x, 128, ue8m0)
    floor = np.float32(np.float32(1e-10) / np.float32(448.0))
    if ue8m0:
        floor = np.float32(2.0 ** -42)
    assert np.all(s[1] == floor) and s[2, 1] == floor
    assert np.all(q[1] == 0) and np.all(q[2, 128:256] == 0)
    assert np.all(s[0] > floor)


def test_group_scales_follow_their_group():
    x = inp.normal_bf16(5, (2, 512))
    _, s0 = oracle.group_quant(x, 128)
    x2 = x.copy()
    x2[1, 300] = inp.to_bf16_bits(np.array([1000.0]))[0]          # spike in group 2 of row 1
    _, s1 = oracle.group_quant(x2, 128)
    changed = np.argwhere(s0 != s1)
    assert changed.tolist() == [[1, 2]]
    assert s1[1, 2] == np.float32(np.float32(1000.0) / np.float32(448.0))


def _expand(spec):
    return np.concatenate([np.full(n, v, np.float32) for v, n in spec])


def _case_arrays(c, key):
    if key in c:
        return np.array(c[key], np.float32)
    return _expand(c[key + "_fill"])[None, :]


def test_rmsnorm_closed_forms(golden):
    for c in golden["rmsnorm_quant"]["cases"]:
        x = _case_arrays(c, "x")
        w = np.array(c["w"], np.float32) if "w" in c else np.full(x.shape[1], c["w_fill"], np.float32)
        q, s, y = oracle.rmsnorm_quant(inp.to_bf16_bits(x), inp.to_bf16_bits(w), c["eps"],
                                       c["group"], want_y=True)
        np.testing.assert_array_equal(y, _case_arrays(c, "y"), err_msg=c["name"])
        if "codes" in c:
            np.testing.assert_array_equal(q, np.array(c["codes"], np.uint8), err_msg=c["name"])
        else:
            for v, n in c["codes_fill"]:
                assert np.all(q == v) and q.size == n
        want_s = [np.float32(np.float32(a) / np.float32(448.0)) for a in c["scale_num"]]
        np.testing.assert_array_equal(s[0], np.array(want_s, np.float32), err_msg=c["name"])


def test_silu_mul_closed_forms(golden):
    for c in golden["silu_mul_quant"]["cases"]:
        x = np.array(c["x"], np.float32)
        q, s, y = oracle.silu_mul_quant(inp.to_bf16_bits(x), c["group"], want_y=True)
        np.testing.assert_array_equal(y, np.array(c["y"], np.float32), err_msg=c["name"])
        np.testing.assert_array_equal(q, np.array(c["codes"], np.uint8), err_msg=c["name"])
        want_s = [np.float32(np.float32(a) / np.float32(448.0)) for a in c["scale_num"]]
        np.testing.assert_array_equal(s[0], np.array(want_s, np.float32), err_msg=c["name"])


def test_rmsnorm_constant_rows_saturate():
    # w = 1, each row constant c: y = bf16(c / sqrt(c^2 + eps)) -> +-1 for |c| >> sqrt(eps);
    # every element equals the amax -> +-448.
    H = 256
    vals = np.array([1.0, -2.0, 37.5, -0.25], np.float32)
    x = np.repeat(vals[:, None], H, 1)
    w = np.ones(H, np.float32)
    for g in (128, H):
        q, s, y = oracle.rmsnorm_quant(inp.to_bf16_bits(x), inp.to_bf16_bits(w), 1e-6, g,
                                       want_y=True)
        np.testing.assert_array_equal(y, np.sign(x))
        np.testing.assert_array_equal(q, np.where(x > 0, 0x7E, 0xFE).astype(np.uint8))
        assert np.all(s == np.float32(np.float32(1.0) / np.float32(448.0)))


def test_silu_large_gate_is_identity():
    g_ = np.array([20.0, 32.0, 100.0, 250.0], np.float32)
    u = np.array([1.0, -3.0, 0.5, 2.0], np.float32)
    x = np.concatenate([g_, u])[None, :]
    _, _, y = oracle.silu_mul_quant(inp.to_bf16_bits(x), 4, want_y=True)
    np.testing.assert_array_equal(y[0], g_ * u)
    x0 = np.array([[0.0, 0.0, 5.0, -7.0]], np.float32)               # gate 0 -> y = 0
    _, _, y0 = oracle.silu_mul_quant(inp.to_bf16_bits(x0), 2, want_y=True)
    assert np.all(y0 == 0)


@pytest.mark.parametrize("fn", ["rmsnorm", "silu"])
@pytest.mark.parametrize("ue8m0", [False, True])
def test_fused_ops_quantize_their_y(fn, ue8m0):
    # The fused ops must quantize exactly the y they produce: re-quantizing the
    # returned y with the plain group quant gives the same codes and scales.
    M, L = 7, 512
    if fn == "rmsnorm":
        x = inp.heavy_tailed_bf16(6, M, L)
        w = inp.rms_weight_bf16(7, L)
        q, s, y = oracle.rmsnorm_quant(x, w, 1e-6, 128, ue8m0, want_y=True)
    else:
        x = inp.normal_bf16(8, (M, 2 * L), std=2.0)
        q, s, y = oracle.silu_mul_quant(x, 128, ue8m0, want_y=True)
    q2, s2 = oracle.group_quant(inp.to_bf16_bits(y), 128, ue8m0)
    np.testing.assert_array_equal(q, q2)
    np.testing.assert_array_equal(s, s2)


# ------------------------------------------------------------ residual add + RMSNorm quant
def test_add_rmsnorm_quant_reduces_to_rmsnorm_quant():
    # residual 0: the sum is x itself, so everything equals rmsnorm_quant(x)
    x = inp.heavy_tailed_bf16(91, 5, 512)
    w = inp.rms_weight_bf16(92, 512)
    zero = np.zeros_like(x)
    for g in (128, 512):
        for ue in (False, True):
            q, s, r = oracle.add_rmsnorm_quant(x, zero, w, 1e-6, g, ue)
            q0, s0 = oracle.rmsnorm_quant(x, w, 1e-6, g, ue)
            np.testing.assert_array_equal(r, x)
            np.testing.assert_array_equal(q, q0)
            np.testing.assert_array_equal(s, s0)


def test_add_rmsnorm_quant_cancelling_residual():
    # residual = -x: the sum is +0 everywhere -> floored scale, all codes 0
    x = inp.heavy_tailed_bf16(93, 3, 256)
    q, s, r = oracle.add_rmsnorm_quant(x, x ^ np.uint16(0x8000), inp.rms_weight_bf16(94, 256), 1e-6, 128)
    assert np.all((r & 0x7FFF) == 0)
    assert np.all(q & 0x7F == 0)
    np.testing.assert_array_equal(s, np.float32(np.float32(1e-10) / np.float32(448.0)))


def test_add_rmsnorm_quant_sum_rounding_hand_cases():
    # bf16 has 8 significant bits (ulp(1) = 2^-7); ties of the sum go to the even significand:
    #   1 + 2^-8          halfway between 1 and 1 + 2^-7          -> 1.0
    #   1 + 3*2^-8        halfway between 1 + 2^-7 and 1 + 2^-6   -> 1 + 2^-6
    #   1 + 2^-8 + 2^-15  just above the first midpoint           -> 1 + 2^-7
    x = inp.to_bf16_bits(np.array([[1.0, 1.0, 1.0] + [0.0] * 125]))
    r = inp.to_bf16_bits(np.array([[2.0 ** -8, 3 * 2.0 ** -8, 2.0 ** -8 + 2.0 ** -15] + [0.0] * 125]))
    _, _, h = oracle.add_rmsnorm_quant(x, r, inp.to_bf16_bits(np.ones(128)), 0.0, 128)
    got = inp.bf16_bits_to_f32(h[0, :3])
    np.testing.assert_array_equal(got, np.array([1.0, 1.0 + 2.0 ** -6, 1.0 + 2.0 ** -7], np.float32))


def test_add_rmsnorm_quant_matches_the_unfused_chain():
    # the fused op equals: torch's bf16 add (round to nearest even), then rmsnorm_quant
    import torch
    x = inp.heavy_tailed_bf16(95, 7, 1024)
    r = inp.normal_bf16(96, (7, 1024), std=4.0)
    w = inp.rms_weight_bf16(97, 1024)
    tb = lambda b: torch.from_numpy(b.view(np.int16)).view(torch.bfloat16)
    h = (tb(x) + tb(r)).view(torch.int16).numpy().view(np.uint16)
    q, s, r_out = oracle.add_rmsnorm_quant(x, r, w, 1e-6, 128)
    q0, s0 = oracle.rmsnorm_quant(h, w, 1e-6, 128)
    np.testing.assert_array_equal(r_out, h)
    np.testing.assert_array_equal(q, q0)
    np.testing.assert_array_equal(s, s0)
