"""GPU parity of the E8M0 (packed UE8M0) path against the oracle.

The quant ops' packed mode (ue8m0 = "packed") must match the oracle bit for
bit: codes and E8M0 scale bytes (the fused ops within their tolerance, which
for bytes means identical).  The block-scaled GEMM (tcgen05 kind::mxf8f6f4
with hardware block scaling) must meet the GEMM tolerance against the fp64
reference on the decoded scales, for every variant it runs (Swap-AB tiles,
128-, 224- and 256-column tiles, split-K, stream-K) on shapes with ragged M and N
tails, and on the config shapes through the automatic variant choice.
"""
import numpy as np
import pytest
import torch

import fp8q_inputs as inp
import oracle
from helpers import (assert_fused_quant_close, bf16_to_np, codes_np, config_rows,
                     gemm_tolerance_check, to_dev_bf16, to_dev_codes)

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import fp8_quantized_linear_rms_b200 as fq   # fails loudly if libfp8q.so is missing


@pytest.fixture(autouse=True)
def _auto_variant():
    yield
    if torch.cuda.is_available():
        fq.fp8q_force_gemm_variant()
        assert fq.fp8q_last_device_status() == fq.OK


def _random_e8m0(seed, shape, lo=112, hi=132):
    return np.random.default_rng(seed).integers(lo, hi, size=shape).astype(np.uint8)


def _run_e8(a, b, sa, sb, layout="row_major"):
    M, K = a.shape
    N = b.shape[0]
    ws = fq.make_workspace(M, N, K, 2)
    sa_d = torch.from_numpy(np.ascontiguousarray(sa.T if layout == "group_major" else sa)).cuda()
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    fq.fp8q_scaled_mm_blockwise_e8m0(to_dev_codes(a), to_dev_codes(b), sa_d,
                                     torch.from_numpy(sb).cuda(), a_scale_layout=layout, y=y,
                                     workspace=ws)
    torch.cuda.synchronize()
    return bf16_to_np(y)


def test_e8m0_gemm_one_tile():
    # the smallest case: one 128 x 224 tile and a 32-column tail tile, two K blocks
    M, N, K = 128, 256, 256
    a = inp.random_e4m3_codes(1, (M, K))
    b = inp.random_e4m3_codes(2, (N, K))
    sa, sb = _random_e8m0(3, (M, K // 128)), _random_e8m0(4, (N // 128, K // 128))
    y = _run_e8(a, b, sa, sb, "group_major")
    y_ref, ad = oracle.scaled_mm_blockwise_e8m0(a, b, sa, sb)
    gemm_tolerance_check(y, y_ref, ad, "e8m0 one tile")


E8_VARIANTS = [(0, 128), (0, 224), (0, 256), (1, 16), (1, 32), (1, 64), (1, 128)]


@pytest.mark.parametrize("split", [0, 1, 3])
@pytest.mark.parametrize("swap,bn", E8_VARIANTS)
@pytest.mark.parametrize("M,N,K", [(1, 256, 384), (100, 384, 512), (260, 640, 1024)])
def test_e8m0_gemm_variants(M, N, K, swap, bn, split):
    a = inp.random_e4m3_codes(M * 17 + K, (M, K))
    b = inp.random_e4m3_codes(N * 19 + K, (N, K))
    sa, sb = _random_e8m0(M + 5, (M, K // 128)), _random_e8m0(N + 6, (N // 128, K // 128))
    fq.fp8q_force_gemm_variant(swap, split, bn)
    y = _run_e8(a, b, sa, sb)
    y_ref, ad = oracle.scaled_mm_blockwise_e8m0(a, b, sa, sb)
    gemm_tolerance_check(y, y_ref, ad, f"e8m0 swap={swap} bn={bn} split={split}")


def test_e8m0_gemm_extreme_exponents_and_determinism():
    # scales spanning 2^-40 .. 2^20 (products still normal in fp32); reruns bit-identical
    M, N, K = 200, 512, 768
    a = inp.random_e4m3_codes(61, (M, K))
    b = inp.random_e4m3_codes(62, (N, K))
    sa, sb = _random_e8m0(63, (M, K // 128), 87, 147), _random_e8m0(64, (N // 128, K // 128), 100, 140)
    y0 = _run_e8(a, b, sa, sb)
    y1 = _run_e8(a, b, sa, sb)
    assert np.array_equal(y0.view(np.uint32), y1.view(np.uint32))
    y_ref, ad = oracle.scaled_mm_blockwise_e8m0(a, b, sa, sb)
    gemm_tolerance_check(y0, y_ref, ad, "e8m0 extreme exponents")


@pytest.mark.parametrize("op", ["group", "rms", "silu"])
@pytest.mark.parametrize("layout", ["row_major", "group_major"])
def test_packed_quant_bit_exact(op, layout):
    M, L = 37, 4096
    for g in (128, L):
        if op == "group":
            x = inp.heavy_tailed_bf16(71, M, L)
            q_ref, s_ref = oracle.group_quant(x, g, "packed")
            q, s = fq.fp8q_group_quant(to_dev_bf16(x), g, "packed", scale_layout=layout)
        elif op == "rms":
            x = inp.heavy_tailed_bf16(72, M, L)
            w = inp.rms_weight_bf16(73, L)
            q_ref, s_ref = oracle.rmsnorm_quant(x, w, 1e-6, g, "packed")
            q, s = fq.fp8q_rmsnorm_quant(to_dev_bf16(x), to_dev_bf16(w[None, :])[0], 1e-6, g,
                                         "packed", scale_layout=layout)
        else:
            x = inp.normal_bf16(74, (M, 2 * L), std=3.0)
            q_ref, s_ref = oracle.silu_mul_quant(x, g, "packed")
            q, s = fq.fp8q_silu_mul_quant(to_dev_bf16(x), g, "packed", scale_layout=layout)
        torch.cuda.synchronize()
        assert s.dtype == torch.uint8
        sg = s.cpu().numpy()
        sg = sg.T.copy() if layout == "group_major" else sg
        if op == "group":
            np.testing.assert_array_equal(codes_np(q), q_ref)
            np.testing.assert_array_equal(sg, s_ref)
        else:
            # fused ops: the scale bytes must be identical (a power of two within
            # 1e-5 relative is the same power of two), codes within the fused tolerance
            np.testing.assert_array_equal(sg, s_ref)
            assert_fused_quant_close(codes_np(q), np.zeros(1), q_ref, np.zeros(1), f"{op} packed")


def _e8m0_weights(seed, N, K):
    """Seeded W ~ N(0, 0.02) in 128x128 blocks with power-of-two scales, quantized
    by the oracle: codes and E8M0 bytes [N/128, K/128]."""
    w = inp.weight_bf16(seed, N, K)
    wf = inp.bf16_bits_to_f32(w).reshape(N // 128, 128, K // 128, 128)
    s = oracle.scale(np.abs(wf).max(axis=(1, 3)).astype(np.float32), True)
    q = oracle.e4m3_encode((wf / s[:, None, :, None]).astype(np.float32)).reshape(N, K)
    return q, oracle.e8m0_encode(s)


QWEN8 = inp.linear_shapes(inp.QWEN3_8B)
QWEN32 = inp.linear_shapes(inp.QWEN3_32B)


def _check_config_e8(M, N, K, seed):
    x = inp.heavy_tailed_bf16(seed, M, K)
    a, sa = oracle.group_quant(x, 128, "packed")
    b, sb = _e8m0_weights(N * 3 + K, N, K)
    y = _run_e8(a, b, sa, sb, "group_major")
    rows = config_rows(M, seed + 1)
    y_ref, ad = oracle.scaled_mm_blockwise_e8m0(a, b, sa, sb, rows)
    gemm_tolerance_check(y[rows], y_ref, ad, f"e8m0 M={M} N={N} K={K} "
                         f"{fq.fp8q_select_gemm_variant(M, N, K, 2)}")


@pytest.mark.parametrize("M", [1, 32, 256, 4096])
@pytest.mark.parametrize("layer", ["qkv", "o", "gate_up", "down"])
def test_config_qwen3_8b_e8m0(M, layer):
    K, N = QWEN8[layer]
    _check_config_e8(M, N, K, 1100 + M)


@pytest.mark.parametrize("M", [1, 64, 8192])
@pytest.mark.parametrize("layer", ["qkv", "o", "gate_up", "down"])
def test_config_qwen3_32b_e8m0(M, layer):
    K, N = QWEN32[layer]
    _check_config_e8(M, N, K, 1200 + M)


def test_e8m0_chain_matches_fp32_scale_chain():
    # RMSNorm -> packed E8M0 quant -> E8M0 GEMM equals the same chain with the
    # power-of-two scales kept in fp32 through the fp32-scale blockwise GEMM
    M, H, N = 300, 4096, 2048
    x = to_dev_bf16(inp.heavy_tailed_bf16(81, M, H))
    w = to_dev_bf16(inp.rms_weight_bf16(82, H)[None, :])[0]
    bq, sb8 = _e8m0_weights(83, N, H)
    qa8, sa8 = fq.fp8q_rmsnorm_quant(x, w, 1e-6, 128, "packed", scale_layout="group_major")
    qa1, sa1 = fq.fp8q_rmsnorm_quant(x, w, 1e-6, 128, True, scale_layout="group_major")
    assert torch.equal(qa8.view(torch.uint8), qa1.view(torch.uint8))
    assert torch.equal(torch.pow(2.0, sa8.float() - 127.0), sa1)
    y8 = fq.fp8q_scaled_mm_blockwise_e8m0(qa8, to_dev_codes(bq), sa8, torch.from_numpy(sb8).cuda(),
                                          a_scale_layout="group_major")
    sbf = torch.from_numpy(oracle.e8m0_decode(sb8).astype(np.float32)).cuda()
    y1 = fq.fp8q_scaled_mm_blockwise(qa1, to_dev_codes(bq), sa1, sbf, a_scale_layout="group_major")
    torch.cuda.synchronize()
    a_np = codes_np(qa8)
    y_ref, ad = oracle.scaled_mm_blockwise_e8m0(a_np, bq, sa8.cpu().numpy().T.copy(), sb8)
    gemm_tolerance_check(bf16_to_np(y8), y_ref, ad, "e8m0 chain")
    gemm_tolerance_check(bf16_to_np(y1), y_ref, ad, "fp32 pow2 chain")
