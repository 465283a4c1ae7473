"""GPU parity of the W8A8_INT8 path against the oracle.

Standalone int8 quant must match the oracle bit for bit (codes and scales);
the producer-fused int8 ops meet the fused tolerance (>= 99.9% identical
codes, the rest within one integer step, scales within 1e-5 relative); the
int8 GEMM (tcgen05 kind::i8, exact integer sums) meets the GEMM tolerance
against the oracle's exact integer reference, for every variant it runs and
on the Qwen3 layer shapes through the automatic variant choice.
"""
import numpy as np
import pytest
import torch

import fp8q_inputs as inp
import oracle
from helpers import bf16_to_np, config_rows, gemm_tolerance_check, to_dev_bf16

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import fp8_quantized_linear_rms_b200 as fq   # fails loudly if libfp8q.so is missing


@pytest.fixture(autouse=True)
def _auto_variant():
    yield
    if torch.cuda.is_available():
        fq.fp8q_force_gemm_variant()
        assert fq.fp8q_last_device_status() == fq.OK


def _i8(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy()


def _fused_close_i8(q, s, q_ref, s_ref, what):
    np.testing.assert_allclose(s, s_ref, rtol=1e-5, atol=0, err_msg=what)
    d = q.astype(np.int32) - q_ref.astype(np.int32)
    n = int((d != 0).sum())
    assert n <= 1e-3 * q_ref.size, f"{what}: {n} codes differ"
    assert np.abs(d).max(initial=0) <= 1, f"{what}: a code moved by more than one step"
    return n


@pytest.mark.parametrize("per_token", [False, True])
@pytest.mark.parametrize("M,K", [(1, 128), (37, 4096), (130, 5120), (2, 25600)])
def test_group_quant_i8_bit_exact(M, K, per_token):
    x = inp.heavy_tailed_bf16(8000 + M + K, M, K)
    g = K if per_token else 128
    q_ref, s_ref = oracle.group_quant_i8(x, g)
    q, s = fq.fp8q_group_quant_i8(to_dev_bf16(x), g)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(_i8(q), q_ref)
    np.testing.assert_array_equal(s.cpu().numpy(), s_ref)


def test_group_quant_i8_edge_values_and_ties():
    # exact halves after division (y/s = k + 1/2 with s a power of two: amax = 127 * 2^e),
    # zeros, huge and tiny rows
    K = 256
    t = np.arange(K) - 128.0
    rows = [np.concatenate([[127.0], t[1:] + 0.5]), np.zeros(K), np.full(K, 3e38), np.full(K, 1e-30),
            np.linspace(-1e4, 1e4, K)]
    x = inp.to_bf16_bits(np.stack(rows))
    for g in (128, K):
        q_ref, s_ref = oracle.group_quant_i8(x, g)
        q, s = fq.fp8q_group_quant_i8(to_dev_bf16(x), g)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(_i8(q), q_ref)
        np.testing.assert_array_equal(s.cpu().numpy(), s_ref)


@pytest.mark.parametrize("per_token", [False, True])
@pytest.mark.parametrize("M,L", [(33, 4096), (129, 5120)])
def test_fused_quant_i8(M, L, per_token):
    g = L if per_token else 128
    x = inp.heavy_tailed_bf16(8100 + M + L, M, L)
    w = inp.rms_weight_bf16(8200 + L, L)
    q_ref, s_ref = oracle.rmsnorm_quant_i8(x, w, 1e-6, g)
    q, s = fq.fp8q_rmsnorm_quant_i8(to_dev_bf16(x), to_dev_bf16(w[None, :])[0], 1e-6, g)
    torch.cuda.synchronize()
    _fused_close_i8(_i8(q), s.cpu().numpy(), q_ref, s_ref, "rms i8")
    xs = inp.normal_bf16(8300 + M + L, (M, 2 * L), std=3.0)
    q_ref, s_ref = oracle.silu_mul_quant_i8(xs, g)
    q, s = fq.fp8q_silu_mul_quant_i8(to_dev_bf16(xs), g)
    torch.cuda.synchronize()
    _fused_close_i8(_i8(q), s.cpu().numpy(), q_ref, s_ref, "silu i8")


def _rand_i8(seed, shape):
    return np.random.default_rng(seed).integers(-128, 128, size=shape).astype(np.int8)


def _run(a, b, sa, sb):
    M, K = a.shape
    N = b.shape[0]
    y = fq.fp8q_scaled_mm_i8(torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda(),
                             torch.from_numpy(sa).cuda(), torch.from_numpy(sb).cuda(),
                             workspace=fq.make_workspace(M, N, K, 3))
    torch.cuda.synchronize()
    return bf16_to_np(y)


PT_VARIANTS = [(0, 128), (0, 256), (1, 16), (1, 32), (1, 64), (1, 128)]


@pytest.mark.parametrize("split", [0, 1, 3])
@pytest.mark.parametrize("swap,bn", PT_VARIANTS)
@pytest.mark.parametrize("M,N,K", [(1, 256, 384), (100, 272, 400), (260, 384, 1024)])
def test_scaled_mm_i8_variants(M, N, K, swap, bn, split):
    a, b = _rand_i8(M * 7 + K, (M, K)), _rand_i8(N * 5 + K, (N, K))
    sa, sb = inp.random_scales(M + 1, (M,)), inp.random_scales(N + 2, (N,))
    fq.fp8q_force_gemm_variant(swap, split, bn)
    y = _run(a, b, sa, sb)
    y_ref, ad = oracle.scaled_mm_i8(a, b, sa, sb)
    gemm_tolerance_check(y, y_ref, ad, f"i8 swap={swap} bn={bn} split={split}")


@pytest.mark.parametrize("bn", [128, 256])
@pytest.mark.parametrize("M,N,K", [(1, 256, 384), (300, 640, 768), (1024, 2048, 512)])
def test_scaled_mm_i8_cta_pair(M, N, K, bn):
    a, b = _rand_i8(M * 3 + K, (M, K)), _rand_i8(N * 9 + K, (N, K))
    sa, sb = inp.random_scales(M + 5, (M,)), inp.random_scales(N + 6, (N,))
    fq.fp8q_force_gemm_variant(0, 1, bn, cta_pair=1)
    y = _run(a, b, sa, sb)
    y_ref, ad = oracle.scaled_mm_i8(a, b, sa, sb)
    gemm_tolerance_check(y, y_ref, ad, f"i8 pair bn={bn}")


def test_scaled_mm_i8_extreme_sums():
    # every product +-127*127 (or -128*-128) of one sign: the largest integer sums
    M, N, K = 64, 128, 8192
    a = np.full((M, K), 127, np.int8)
    a[1::2] = -128
    b = np.full((N, K), 127, np.int8)
    b[::3] = -128
    sa, sb = np.full(M, 1e-4, np.float32), np.full(N, 3e-3, np.float32)
    y = _run(a, b, sa, sb)
    y_ref, ad = oracle.scaled_mm_i8(a, b, sa, sb)
    gemm_tolerance_check(y, y_ref, ad, "i8 extreme sums")


QWEN32 = inp.linear_shapes(inp.QWEN3_32B)


@pytest.mark.parametrize("M", [16, 8192])
@pytest.mark.parametrize("layer", ["qkv", "o", "gate_up", "down"])
def test_config_qwen3_32b_i8(M, layer):
    # the W8A8_INT8 linear: per-token int8 activations (quantized by the oracle)
    # times per-channel int8 weights
    K, N = QWEN32[layer]
    x = inp.heavy_tailed_bf16(8400 + M, M, K)
    a, sa = oracle.group_quant_i8(x, K)
    b, sb = oracle.group_quant_i8(inp.weight_bf16(N + K, N, K), K)
    y = _run(a, b, sa.reshape(-1), sb.reshape(-1))
    rows = config_rows(M, 8500 + M)
    y_ref, ad = oracle.scaled_mm_i8(a, b, sa.reshape(-1), sb.reshape(-1), rows)
    gemm_tolerance_check(y[rows], y_ref, ad, f"i8 M={M} {layer} {fq.fp8q_select_gemm_variant(M, N, K, 3)}")
