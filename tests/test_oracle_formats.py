"""Pins of the oracle's number formats against libraries and hand-derived cases.

The e4m3fn encoder is checked exhaustively against ml_dtypes (an independent
library) on every fp32 bit pattern that can round to a nonzero code, and
against torch's CPU cast on a sample; the bf16 rounding against torch and a
double-rounding trap; the scale against hand-derived values.
"""
import ml_dtypes
import numpy as np
import pytest
import torch

import oracle


def _lib_e4m3(v: np.ndarray) -> np.ndarray:
    """Library e4m3fn encode of fp32 values, saturating (clamp first: ml_dtypes maps overflow to NaN)."""
    return np.clip(v, -448.0, 448.0).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)


def test_e4m3_encode_exhaustive_vs_ml_dtypes():
    # Every positive fp32 pattern from 2^-12 up to 464 (all values that do not
    # trivially round to zero, and the whole saturation boundary), both signs.
    lo = np.float32(2.0 ** -12).view(np.uint32)
    hi = np.float32(464.0).view(np.uint32) + 1
    chunk = 1 << 24
    start = int(lo)
    while start < hi:
        stop = min(start + chunk, int(hi))
        v = np.arange(start, stop, dtype=np.uint32).view(np.float32)
        got = oracle.e4m3_encode(v)
        np.testing.assert_array_equal(got, _lib_e4m3(v))
        np.testing.assert_array_equal(oracle.e4m3_encode(-v), got | 0x80)
        start = stop


def test_e4m3_encode_tiny_and_huge():
    g = np.random.default_rng(7)
    tiny = (np.arange(0, int(np.float32(2.0 ** -12).view(np.uint32)), 9973, dtype=np.uint32)
            .view(np.float32))
    np.testing.assert_array_equal(oracle.e4m3_encode(tiny), 0)
    np.testing.assert_array_equal(oracle.e4m3_encode(-tiny), 0x80)   # sign of zero kept
    huge = np.concatenate([g.uniform(464, 3e38, 10000).astype(np.float32),
                           np.array([np.float32(464.0) + np.float32(2.0 ** -14) * 1024,
                                     np.finfo(np.float32).max], np.float32)])
    np.testing.assert_array_equal(oracle.e4m3_encode(huge), 0x7E)
    np.testing.assert_array_equal(oracle.e4m3_encode(-huge), 0xFE)


def test_e4m3_encode_vs_torch_cast_sample():
    g = np.random.default_rng(11)
    v = np.concatenate([g.normal(0, 1, 200000), g.normal(0, 100, 200000),
                        g.uniform(-448, 448, 200000)]).astype(np.float32)
    ref = torch.from_numpy(np.clip(v, -448, 448)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(oracle.e4m3_encode(v), ref)


def test_e4m3_encode_hand_cases(golden):
    for c in golden["e4m3_encode"]["cases"]:
        assert int(oracle.e4m3_encode(np.array([c["x"]]))[0]) == c["code"], c


def test_e4m3_decode_all_codes_vs_ml_dtypes():
    codes = np.arange(256, dtype=np.uint8)
    got = oracle.e4m3_decode(codes)
    ref = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    nan = np.isnan(ref)
    assert set(np.nonzero(nan)[0].tolist()) == {0x7F, 0xFF}
    np.testing.assert_array_equal(np.isnan(got), nan)
    np.testing.assert_array_equal(got[~nan], ref[~nan])
    # encode(decode(c)) == c for every finite code
    np.testing.assert_array_equal(oracle.e4m3_encode(got[~nan].astype(np.float32)), codes[~nan])


def test_bf16_round_vs_torch_on_fp32_values():
    g = np.random.default_rng(3)
    v = np.concatenate([g.normal(0, 1, 300000), g.standard_t(3, 300000) * 50,
                        np.ldexp(g.uniform(1, 2, 20000), g.integers(-140, -120, 20000))])
    v = v.astype(np.float32).astype(np.float64)       # exactly fp32-representable
    ref = torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16).float().numpy()
    np.testing.assert_array_equal(oracle.bf16_round(v), ref)


def test_bf16_round_single_rounding():
    # 1 + 2^-8 + 2^-30 lies just above the midpoint of 1 and 1 + 2^-7; a
    # detour through fp32 would land exactly on the midpoint and round to 1.
    assert oracle.bf16_round(np.array([1.0 + 2.0 ** -8 + 2.0 ** -30]))[0] == np.float32(1.0078125)
    assert oracle.bf16_round(np.array([1.0 + 2.0 ** -8]))[0] == np.float32(1.0)        # tie -> even
    assert oracle.bf16_round(np.array([1.0 + 3 * 2.0 ** -8]))[0] == np.float32(1.015625)  # tie -> even
    assert oracle.bf16_round(np.array([-(1.0 + 2.0 ** -8 + 2.0 ** -30)]))[0] == np.float32(-1.0078125)


def test_scale_hand_cases(golden):
    for c in golden["scale"]["cases"]:
        got = float(oracle.scale(np.array([c["amax"]], np.float32), bool(c["ue8m0"]))[0])
        assert got == c["scale"], c
    floor = np.float32(np.float32(1e-10) / np.float32(448.0))
    assert oracle.scale(np.array([0.0], np.float32))[0] == floor
    assert oracle.scale(np.array([1e-12], np.float32))[0] == floor


@pytest.mark.parametrize("ue8m0", [False, True])
def test_scale_properties(ue8m0):
    g = np.random.default_rng(5)
    amax = np.abs(np.concatenate([g.standard_t(2, 100000) * 10, g.uniform(0, 1e-9, 1000)])
                  ).astype(np.float32)
    s = oracle.scale(amax, ue8m0).astype(np.float64)
    base = (np.maximum(amax, np.float32(1e-10)) / np.float32(448.0)).astype(np.float64)
    if not ue8m0:
        np.testing.assert_array_equal(s, base)
    else:
        m, _ = np.frexp(s)
        assert np.all(m == 0.5)                       # powers of two
        assert np.all(s >= base) and np.all(s < 2 * base)


# ------------------------------------------------------------------ E8M0
def test_e8m0_decode_all_bytes_vs_ml_dtypes():
    # Every byte, against an independent library's E8M0 type (2^(b-127), 255 = NaN).
    b = np.arange(256, dtype=np.uint8)
    ref = b.view(ml_dtypes.float8_e8m0fnu).astype(np.float64)
    got = oracle.e8m0_decode(b)
    np.testing.assert_array_equal(np.isnan(got), np.isnan(ref))
    np.testing.assert_array_equal(got[:255], ref[:255])
    assert got[127] == 1.0 and got[0] == 2.0 ** -127 and got[254] == 2.0 ** 127


def test_e8m0_encode_powers_of_two_and_rejects():
    # Every power of two an fp32 holds in [2^-126, 2^127] (fp32 normals; 2^-127 is an
    # fp32 subnormal, also a power of two) encodes to its exponent + 127, as the
    # library's cast does; anything that is not a power of two gives 255.
    k = np.arange(-127, 128)
    s = np.ldexp(np.float32(1.0), k).astype(np.float32)
    got = oracle.e8m0_encode(s)
    np.testing.assert_array_equal(got, (k + 127).astype(np.uint8))
    np.testing.assert_array_equal(got, s.astype(ml_dtypes.float8_e8m0fnu).view(np.uint8))
    bad = np.array([0.0, -1.0, 3.0, 1.5, np.inf, np.nan, 2.0 ** -128, 0.75], np.float32)
    np.testing.assert_array_equal(oracle.e8m0_encode(bad), 0xFF)


@pytest.mark.parametrize("op", ["group", "rms", "silu"])
def test_packed_ue8m0_scales_are_the_ue8m0_exponents(op):
    # The packed mode stores the byte of the UE8M0 scale: same codes as ue8m0=1,
    # and every byte decodes to exactly the fp32 power-of-two scale.
    import fp8q_inputs as inp
    x = inp.heavy_tailed_bf16(31, 9, 512)
    w = inp.rms_weight_bf16(32, 512)
    for g in (128, 512):
        if op == "group":
            q1, s1 = oracle.group_quant(x, g, True)
            qp, sp = oracle.group_quant(x, g, "packed")
        elif op == "rms":
            q1, s1 = oracle.rmsnorm_quant(x, w, 1e-6, g, True)
            qp, sp = oracle.rmsnorm_quant(x, w, 1e-6, g, "packed")
        else:
            xs = inp.heavy_tailed_bf16(33, 9, 1024)
            q1, s1 = oracle.silu_mul_quant(xs, g, True)
            qp, sp = oracle.silu_mul_quant(xs, g, "packed")
        assert sp.dtype == np.uint8 and sp.shape == s1.shape
        np.testing.assert_array_equal(qp, q1)
        np.testing.assert_array_equal(sp.view(ml_dtypes.float8_e8m0fnu).astype(np.float32), s1)


def test_packed_ue8m0_hand_cases():
    # amax 448 -> s = 1 -> byte 127; amax 1 -> 1/448 rounds up to 2^-8 -> 119;
    # amax 0 -> floored 1e-10/448 ~ 2^-42.03 rounds up to 2^-42 -> 85;
    # amax 3.5 -> 3.5/448 = 2^-7 exactly -> kept -> 120.
    import fp8q_inputs as inp
    rows = np.zeros((4, 128))
    rows[0, 5] = 448.0
    rows[1, 7] = -1.0
    rows[3, 0] = 3.5
    _, sp = oracle.group_quant(inp.to_bf16_bits(rows), 128, "packed")
    np.testing.assert_array_equal(sp.reshape(-1), np.array([127, 119, 85, 120], np.uint8))
