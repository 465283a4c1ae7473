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
