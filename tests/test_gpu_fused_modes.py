"""The two arithmetic modes of the producer-fused quant ops against the oracle.

Fast mode (the default) computes y in fp32 and recomputes exactly the
elements that can decide a group's amax: its scales must equal the
definition's bit for bit and its codes meet the fused tolerance (>= 99.9%
identical, the rest within one step).  Exact mode must equal the definition
bit for bit in codes and scales.  Cases: the config-5 row lengths with
heavy-tailed activations, both group sizes, int8 codes, and the rows that
send the fast path to its exact routes (sums of squares out of fp32 range,
gates below -85 next to huge up values).
"""
import numpy as np
import pytest
import torch

import fp8q_inputs as inp
import oracle
from helpers import assert_fused_quant_close, codes_np, fused_quant_exact, to_dev_bf16

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import fp8_quantized_linear_rms_b200 as fq   # fails loudly if libfp8q.so is missing


def _rms(x, w, g, ue8m0=False):
    q, s = fq.fp8q_rmsnorm_quant(to_dev_bf16(x), to_dev_bf16(w[None, :])[0], 1e-6, g, ue8m0)
    torch.cuda.synchronize()
    return codes_np(q), s.cpu().numpy()


def _silu(x, g, ue8m0=False):
    q, s = fq.fp8q_silu_mul_quant(to_dev_bf16(x), g, ue8m0)
    torch.cuda.synchronize()
    return codes_np(q), s.cpu().numpy()


@pytest.mark.parametrize("per_token", [True, False])
@pytest.mark.parametrize("M,H", [(37, 5120), (300, 4096), (9, 16384), (5, 20480)])
def test_rmsnorm_modes(M, H, per_token):
    x = inp.heavy_tailed_bf16(8100 + M + H, M, H)
    w = inp.rms_weight_bf16(8200 + H, H)
    g = H if per_token else 128
    q_ref, s_ref = oracle.rmsnorm_quant(x, w, 1e-6, g)
    q, s = _rms(x, w, g)                                   # fast (default)
    np.testing.assert_array_equal(s, s_ref)
    n = assert_fused_quant_close(q, s, q_ref, s_ref, "rmsnorm fast")
    print(f"rmsnorm fast M={M} H={H} g={g}: {n} of {q_ref.size} codes differ")
    with fused_quant_exact(True):
        q, s = _rms(x, w, g)
    np.testing.assert_array_equal(s, s_ref)
    np.testing.assert_array_equal(q, q_ref)


@pytest.mark.parametrize("per_token", [True, False])
@pytest.mark.parametrize("M,I", [(33, 25600), (130, 12288), (65, 4096)])
def test_silu_mul_modes(M, I, per_token):
    x = inp.heavy_tailed_bf16(8300 + M + I, M, 2 * I)
    g = I if per_token else 128
    q_ref, s_ref = oracle.silu_mul_quant(x, g)
    q, s = _silu(x, g)
    np.testing.assert_array_equal(s, s_ref)
    n = assert_fused_quant_close(q, s, q_ref, s_ref, "silu fast")
    print(f"silu fast M={M} I={I} g={g}: {n} of {q_ref.size} codes differ")
    with fused_quant_exact(True):
        q, s = _silu(x, g)
    np.testing.assert_array_equal(s, s_ref)
    np.testing.assert_array_equal(q, q_ref)


def test_add_rmsnorm_modes():
    M, H = 70, 5120
    x = inp.heavy_tailed_bf16(8401, M, H)
    r = inp.heavy_tailed_bf16(8402, M, H)
    w = inp.rms_weight_bf16(8403, H)
    for g in (H, 128):
        q_ref, s_ref, r_ref = oracle.add_rmsnorm_quant(x, r, w, 1e-6, g)
        for exact in (False, True):
            rd = to_dev_bf16(r)
            with fused_quant_exact(exact):
                q, s = fq.fp8q_add_rmsnorm_quant(to_dev_bf16(x), rd, to_dev_bf16(w[None, :])[0], 1e-6, g)
                torch.cuda.synchronize()
            np.testing.assert_array_equal(rd.view(torch.int16).cpu().numpy().view(np.uint16), r_ref)
            np.testing.assert_array_equal(s.cpu().numpy(), s_ref)
            if exact:
                np.testing.assert_array_equal(codes_np(q), q_ref)
            else:
                assert_fused_quant_close(codes_np(q), s.cpu().numpy(), q_ref, s_ref, "add+rms fast")


@pytest.mark.parametrize("ue8m0", [False, True])
def test_rmsnorm_fast_exact_routes(ue8m0):
    # rows whose sum of squares leaves the fp32 range of the fast sum (squares
    # of 1e30 overflow; a row of 1e-30 values sums below 2^-100), a row mixing
    # both, and ordinary rows between them: scales exact, codes within tolerance
    H = 2048
    rng = np.random.default_rng(8500)
    rows = [rng.normal(0, 1e30, H), rng.normal(0, 1e-30, H),
            np.where(np.arange(H) % 7 == 0, 3e25, rng.normal(0, 1e-20, H)),
            rng.normal(0, 1.0, H), rng.standard_t(3, H) * 1e-3]
    x = inp.to_bf16_bits(np.stack(rows))
    w = inp.rms_weight_bf16(8501, H)
    for g in (H, 128):
        q_ref, s_ref = oracle.rmsnorm_quant(x, w, 1e-6, g, ue8m0)
        q, s = _rms(x, w, g, ue8m0)
        np.testing.assert_array_equal(s, s_ref)
        assert_fused_quant_close(q, s, q_ref, s_ref, "rmsnorm fast, exact routes")


@pytest.mark.parametrize("I", [1024, 25600])
def test_silu_fast_low_gates_with_huge_up(I):
    # a gate below -85 next to a huge up value makes a row's amax although its
    # fp32 exponential overflows: the fast path sends such chunks to the exact
    # arithmetic, so the scales stay exact
    rng = np.random.default_rng(8600 + I)
    g = rng.normal(0.0, 1e-3, size=(3, I))
    u = rng.normal(0.0, 1e-3, size=(3, I))
    g[0, 17], u[0, 17] = -89.0, 2.0 ** 120          # silu(g) u ~ -0.27, the row's amax
    g[1, I - 3], u[1, I - 3] = -95.0, -(2.0 ** 126)
    g[2, 0], u[2, 0] = -86.0, 2.0 ** 118
    x = inp.to_bf16_bits(np.concatenate([g, u], axis=1))
    for gs in (I, 128):
        q_ref, s_ref = oracle.silu_mul_quant(x, gs)
        q, s = _silu(x, gs)
        np.testing.assert_array_equal(s, s_ref)
        assert_fused_quant_close(q, s, q_ref, s_ref, "silu fast, low gates")


@pytest.mark.parametrize("op", ["rmsnorm", "silu"])
def test_int8_fast_mode(op):
    M, L = 41, 5120
    for g in (L, 128):
        if op == "rmsnorm":
            x = inp.heavy_tailed_bf16(8700, M, L)
            w = inp.rms_weight_bf16(8701, L)
            q_ref, s_ref = oracle.rmsnorm_quant_i8(x, w, 1e-6, g)
            q, s = fq.fp8q_rmsnorm_quant_i8(to_dev_bf16(x), to_dev_bf16(w[None, :])[0], 1e-6, g)
        else:
            x = inp.heavy_tailed_bf16(8702, M, 2 * L)
            q_ref, s_ref = oracle.silu_mul_quant_i8(x, g)
            q, s = fq.fp8q_silu_mul_quant_i8(to_dev_bf16(x), g)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(s.cpu().numpy(), s_ref)
        qi = q.view(torch.int8).cpu().numpy().astype(np.int32)
        diff = qi != q_ref.astype(np.int32)
        assert diff.sum() <= 1e-3 * q_ref.size, f"{op} i8: {diff.sum()} codes differ"
        assert np.all(np.abs(qi[diff] - q_ref.astype(np.int32)[diff]) <= 1)
