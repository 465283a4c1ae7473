"""GPU parity of the scaled FP8 GEMMs against the oracle's fp64 reference.

Pass condition (per output element): |y - y_ref| <= 2^-8 |y_ref| + 1e-3 sum_k |a_k b_k|,
with y_ref the fp64 sum of the dequantized operands.  Every GEMM variant
(tile width, Swap-AB, Split-K) is forced in turn on shapes that span several
tiles and ragged M / N / K tails and checked in full; the config shapes
(Qwen3-8B / 32B linears, decode and prefill M) run through the automatic
variant choice and are checked on every column of 256 stratified rows (every
256-row tile and both of its 128-row halves) plus every row of the last
256-row tile; decode batches (M <= 256) in full.
"""
import numpy as np
import pytest
import torch

import fp8q_inputs as inp
import oracle
from helpers import (bf16_to_np, config_rows, gemm_tolerance_check, quantized_weights,
                     to_dev_bf16, to_dev_codes)

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import fp8_quantized_linear_rms_b200 as fq   # fails loudly if libfp8q.so is missing

PT_VARIANTS = [(0, 128), (0, 256), (1, 16), (1, 32), (1, 64), (1, 128)]
BW_VARIANTS = [(0, 128), (0, 256), (1, 16), (1, 32), (1, 64), (1, 128)]


@pytest.fixture(autouse=True)
def _auto_variant():
    yield
    if torch.cuda.is_available():
        fq.fp8q_force_gemm_variant()
        assert fq.fp8q_last_device_status() == fq.OK


def _run_pt(a, b, sa, sb, M, N, K):
    ws = fq.make_workspace(M, N, K, False)
    y = fq.fp8q_scaled_mm(to_dev_codes(a), to_dev_codes(b), torch.from_numpy(sa).cuda(),
                          torch.from_numpy(sb).cuda(), workspace=ws)
    torch.cuda.synchronize()
    return bf16_to_np(y)


def _run_bw(a, b, sa, sb, M, N, K, layout="row_major"):
    ws = fq.make_workspace(M, N, K, True)
    sa_d = torch.from_numpy(np.ascontiguousarray(sa.T if layout == "group_major" else sa)).cuda()
    y = fq.fp8q_scaled_mm_blockwise(to_dev_codes(a), to_dev_codes(b), sa_d,
                                    torch.from_numpy(sb).cuda(), a_scale_layout=layout,
                                    workspace=ws)
    torch.cuda.synchronize()
    return bf16_to_np(y)


@pytest.mark.parametrize("split", [0, 1, 3])
@pytest.mark.parametrize("swap,bn", PT_VARIANTS)
@pytest.mark.parametrize("M,N,K", [(1, 256, 384), (100, 272, 400), (260, 384, 1024)])
def test_scaled_mm_variants(M, N, K, swap, bn, split):
    a = inp.random_e4m3_codes(M * 7 + K, (M, K))
    b = inp.random_e4m3_codes(N * 5 + K, (N, K))
    sa = inp.random_scales(M + 1, (M,))
    sb = inp.random_scales(N + 2, (N,))
    fq.fp8q_force_gemm_variant(swap, split, bn)
    y = _run_pt(a, b, sa, sb, M, N, K)
    y_ref, ad = oracle.scaled_mm(a, b, sa, sb)
    gemm_tolerance_check(y, y_ref, ad, f"pt swap={swap} bn={bn} split={split}")


@pytest.mark.parametrize("split", [0, 1, 3])
@pytest.mark.parametrize("swap,bn", BW_VARIANTS)
@pytest.mark.parametrize("M,N,K", [(1, 256, 384), (100, 384, 512), (260, 256, 1024)])
def test_scaled_mm_blockwise_variants(M, N, K, swap, bn, split):
    a = inp.random_e4m3_codes(M * 11 + K, (M, K))
    b = inp.random_e4m3_codes(N * 13 + K, (N, K))
    sa = inp.random_scales(M + 3, (M, K // 128))
    sb = inp.random_scales(N + 4, (N // 128, K // 128))
    fq.fp8q_force_gemm_variant(swap, split, bn)
    y = _run_bw(a, b, sa, sb, M, N, K)
    y_ref, ad = oracle.scaled_mm_blockwise(a, b, sa, sb)
    gemm_tolerance_check(y, y_ref, ad, f"bw swap={swap} bn={bn} split={split}")


# CTA pairs (cta_group::2): 256-row tiles on two SMs; tiny M leaves the odd
# CTA's rows outside the matrix, K tails and many tiles per pair included.
PAIR_SHAPES = [(1, 256, 384), (100, 384, 512), (260, 256, 1024), (600, 640, 768), (1024, 2048, 512)]


@pytest.mark.parametrize("bn", [128, 256])
@pytest.mark.parametrize("M,N,K", PAIR_SHAPES + [(100, 272, 400)])
def test_scaled_mm_cta_pair(M, N, K, bn):
    a = inp.random_e4m3_codes(M * 3 + K, (M, K))
    b = inp.random_e4m3_codes(N * 7 + K, (N, K))
    sa = inp.random_scales(M + 5, (M,))
    sb = inp.random_scales(N + 6, (N,))
    fq.fp8q_force_gemm_variant(0, 1, bn, cta_pair=1)
    y = _run_pt(a, b, sa, sb, M, N, K)
    y_ref, ad = oracle.scaled_mm(a, b, sa, sb)
    gemm_tolerance_check(y, y_ref, ad, f"pt pair bn={bn}")


@pytest.mark.parametrize("layout", ["row_major", "group_major"])
@pytest.mark.parametrize("M,N,K", PAIR_SHAPES)
def test_scaled_mm_blockwise_cta_pair(M, N, K, layout):
    a = inp.random_e4m3_codes(M * 5 + K, (M, K))
    b = inp.random_e4m3_codes(N * 9 + K, (N, K))
    sa = inp.random_scales(M + 7, (M, K // 128))
    sb = inp.random_scales(N + 8, (N // 128, K // 128))
    fq.fp8q_force_gemm_variant(0, 1, 128, cta_pair=1)
    y = _run_bw(a, b, sa, sb, M, N, K, layout)
    y_ref, ad = oracle.scaled_mm_blockwise(a, b, sa, sb)
    gemm_tolerance_check(y, y_ref, ad, f"bw pair {layout}")


def test_cta_pair_determinism_and_canaries():
    # the same output bits on reruns; nothing written outside y's rows
    M, N, K = 300, 512, 1024
    a = to_dev_codes(inp.random_e4m3_codes(91, (M, K)))
    b = to_dev_codes(inp.random_e4m3_codes(92, (N, K)))
    sa = torch.from_numpy(inp.random_scales(93, (M, K // 128))).cuda()
    sb = torch.from_numpy(inp.random_scales(94, (N // 128, K // 128))).cuda()
    fq.fp8q_force_gemm_variant(0, 1, 128, cta_pair=1)
    ys = []
    for _ in range(2):
        big = torch.full((M + 2, N), 12345.0, dtype=torch.bfloat16, device="cuda")
        fq.fp8q_scaled_mm_blockwise(a, b, sa, sb, y=big[1:M + 1])
        torch.cuda.synchronize()
        assert torch.all(big[0] == 12345.0) and torch.all(big[M + 1] == 12345.0)
        ys.append(big[1:M + 1].clone())
    assert torch.equal(ys[0], ys[1])


def test_blockwise_group_major_scales_and_ue8m0():
    M, N, K = 70, 256, 640
    a = inp.random_e4m3_codes(21, (M, K))
    b = inp.random_e4m3_codes(22, (N, K))
    sa = inp.random_pow2_scales(23, (M, K // 128))
    sb = inp.random_pow2_scales(24, (N // 128, K // 128))
    y = _run_bw(a, b, sa, sb, M, N, K, layout="group_major")
    y_ref, ad = oracle.scaled_mm_blockwise(a, b, sa, sb)
    gemm_tolerance_check(y, y_ref, ad, "bw group-major ue8m0")


@pytest.mark.parametrize("per_token,per_channel", [(False, False), (False, True), (True, False)])
def test_scaled_mm_per_tensor_scales(per_token, per_channel):
    M, N, K = 33, 256, 256
    a = inp.random_e4m3_codes(31, (M, K))
    b = inp.random_e4m3_codes(32, (N, K))
    sa = inp.random_scales(33, (M if per_token else 1,))
    sb = inp.random_scales(34, (N if per_channel else 1,))
    y = _run_pt(a, b, sa, sb, M, N, K)
    y_ref, ad = oracle.scaled_mm(a, b, sa, sb)
    gemm_tolerance_check(y, y_ref, ad, "per-tensor scales")


def test_small_k_tail():
    M, N, K = 3, 128, 48                    # K < one 128-deep stage: zero-filled by TMA
    a = inp.random_e4m3_codes(41, (M, K))
    b = inp.random_e4m3_codes(42, (N, K))
    sa = inp.random_scales(43, (M,))
    sb = inp.random_scales(44, (N,))
    for swap, bn in ((0, 128), (1, 16)):
        fq.fp8q_force_gemm_variant(swap, 1, bn)
        y = _run_pt(a, b, sa, sb, M, N, K)
        y_ref, ad = oracle.scaled_mm(a, b, sa, sb)
        gemm_tolerance_check(y, y_ref, ad, f"K tail swap={swap}")


@pytest.mark.parametrize("split", [0, 4])
@pytest.mark.parametrize("blockwise", [False, True])
@pytest.mark.parametrize("swap,bn", [(0, 128), (1, 32)])
def test_output_canaries_and_split_determinism(blockwise, swap, bn, split):
    # y is a view into a larger buffer (extra columns and rows): nothing outside
    # [M, N] may change; split-K results are bit-identical across runs and the
    # workspace is reusable without clearing.
    M, N, K = 45, 256, 1024
    a = inp.random_e4m3_codes(51, (M, K))
    b = inp.random_e4m3_codes(52, (N, K))
    sa = inp.random_scales(53, (M, K // 128) if blockwise else (M,))
    sb = inp.random_scales(54, (N // 128, K // 128) if blockwise else (N,))
    fq.fp8q_force_gemm_variant(swap, split, bn)
    ws = fq.make_workspace(M, N, K, blockwise)
    assert ws is not None
    big = torch.full((M + 3, N + 24), 7.0, dtype=torch.bfloat16, device="cuda")
    y = big[:M, :N]
    outs = []
    for _ in range(3):
        if blockwise:
            fq.fp8q_scaled_mm_blockwise(to_dev_codes(a), to_dev_codes(b), torch.from_numpy(sa).cuda(),
                                        torch.from_numpy(sb).cuda(), y=y, workspace=ws)
        else:
            fq.fp8q_scaled_mm(to_dev_codes(a), to_dev_codes(b), torch.from_numpy(sa).cuda(),
                              torch.from_numpy(sb).cuda(), y=y, workspace=ws)
        torch.cuda.synchronize()
        outs.append(y.clone())
    for o in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16))
    full = big.float().cpu().numpy()
    assert np.all(full[:, N:] == 7.0) and np.all(full[M:, :] == 7.0)
    if blockwise:
        y_ref, ad = oracle.scaled_mm_blockwise(a, b, sa, sb)
    else:
        y_ref, ad = oracle.scaled_mm(a, b, sa, sb)
    gemm_tolerance_check(bf16_to_np(y), y_ref, ad, "canary case")


def test_abi_rejects_bad_arguments():
    a = torch.zeros((4, 256), dtype=torch.uint8, device="cuda")
    s = torch.ones(4, dtype=torch.float32, device="cuda")
    y = torch.empty((4, 256), dtype=torch.bfloat16, device="cuda")
    L = fq.lib
    p = lambda t: t.data_ptr()
    st = torch.cuda.current_stream().cuda_stream
    # N not a multiple of 16
    assert L.fp8q_scaled_mm(p(a), p(a), p(s), 1, p(s), 1, 4, 8, 256, p(y), 256, None, 0, st) == fq.ERR_INVALID_ARG
    # blockwise with K not a multiple of 128
    assert L.fp8q_scaled_mm_blockwise(p(a), p(a), p(s), 1, 4, p(s), 4, 128, 144, p(y), 256, None, 0,
                                      st) == fq.ERR_INVALID_ARG
    # misaligned output
    assert L.fp8q_scaled_mm(p(a), p(a), p(s), 1, p(s), 1, 4, 128, 256, p(y) + 2, 256, None, 0, st) == fq.ERR_INVALID_ARG
    # a split-K shape without its workspace
    fq.fp8q_force_gemm_variant(1, 4, 16)
    assert fq.fp8q_workspace_bytes(4, 256, 1024, False) > 0
    big = torch.zeros((256, 1024), dtype=torch.uint8, device="cuda")
    assert L.fp8q_scaled_mm(p(big), p(big), p(s), 1, p(s), 1, 4, 256, 1024, p(y), 256, None, 0,
                            st) == fq.ERR_INVALID_ARG
    # quant: bad group size, bad ue8m0
    x = torch.zeros((4, 256), dtype=torch.bfloat16, device="cuda")
    assert L.fp8q_group_quant(p(x), 4, 256, 256, 64, 0, p(a), 256, p(s), 1, 1, st) == fq.ERR_INVALID_ARG
    assert L.fp8q_group_quant(p(x), 4, 256, 256, 128, 3, p(a), 256, p(s), 2, 1, st) == fq.ERR_INVALID_ARG
    torch.cuda.synchronize()


# ------------------------------------------------------------ config shapes
def _check_config_gemm(M, N, K, blockwise, seed, act="normal"):
    """Activations quantized by the oracle (1x128 groups or per token), weights
    W ~ N(0, 0.02) quantized by the oracle (128x128 blocks or per channel).
    Checked: every column of 256 stratified rows (every 256-row tile, both
    128-row halves) and of every row of the last 256-row tile."""
    if act == "heavy":
        x = inp.heavy_tailed_bf16(seed, M, K)
    else:
        x = inp.normal_bf16(seed, (M, K))
    b, sb = _weights(N, K, blockwise)
    if blockwise:
        a, sa = oracle.group_quant(x, 128)
    else:
        a, sa = oracle.group_quant(x, K)
        sa = sa.reshape(-1)
        sb = sb.reshape(-1)
    rows = config_rows(M, seed + 2)
    if blockwise:
        y = _run_bw(a, b, sa, sb, M, N, K)
        y_ref, ad = oracle.scaled_mm_blockwise(a, b, sa, sb, rows)
    else:
        y = _run_pt(a, b, sa, sb, M, N, K)
        y_ref, ad = oracle.scaled_mm(a, b, sa, sb, rows)
    v = fq.fp8q_select_gemm_variant(M, N, K, blockwise)
    gemm_tolerance_check(y[rows], y_ref, ad, f"M={M} N={N} K={K} bw={blockwise} {v}")


_WEIGHTS = {}


def _weights(N, K, blockwise):
    key = (N, K, blockwise)
    if key not in _WEIGHTS:
        if len(_WEIGHTS) >= 4:
            _WEIGHTS.clear()
        _WEIGHTS[key] = quantized_weights(N * 7 + K, N, K, blockwise)
    return _WEIGHTS[key]


QWEN8 = inp.linear_shapes(inp.QWEN3_8B)
QWEN32 = inp.linear_shapes(inp.QWEN3_32B)


@pytest.mark.parametrize("M", [1, 16, 128, 2048])
@pytest.mark.parametrize("layer", ["gate_up", "down"])
def test_config_qwen3_8b_per_token_mlp(M, layer):
    K, N = QWEN8[layer]
    _check_config_gemm(M, N, K, False, 700 + M, act="heavy")


@pytest.mark.parametrize("M", [1, 3, 32, 100, 256, 1000, 4096])
@pytest.mark.parametrize("layer", ["qkv", "o", "gate_up", "down"])
def test_config_qwen3_8b_blockwise(M, layer):
    K, N = QWEN8[layer]
    _check_config_gemm(M, N, K, True, 800 + M)


@pytest.mark.parametrize("M", [1, 2, 4, 8, 16, 32, 64])
@pytest.mark.parametrize("layer", ["qkv", "o", "gate_up", "down"])
def test_config_qwen3_32b_decode_blockwise(M, layer):
    K, N = QWEN32[layer]
    _check_config_gemm(M, N, K, True, 900 + M)


@pytest.mark.parametrize("blockwise", [False, True])
@pytest.mark.parametrize("layer", ["qkv", "o", "gate_up", "down"])
def test_config_qwen3_32b_prefill(layer, blockwise):
    K, N = QWEN32[layer]
    _check_config_gemm(8192, N, K, blockwise, 1000, act="heavy")


def test_config_tiny_per_token_linear_chain():
    # x [16, 2048] -> RMSNorm + per-token quant (GPU) -> scaled_mm with a per-channel
    # quantized W [2048, 2048]; compared with the oracle's own chain.
    M, H, N = 16, 2048, 2048
    x = inp.normal_bf16(1, (M, H))
    w = inp.rms_weight_bf16(2, H)
    b, sb = quantized_weights(3, N, H, False)
    qa, sa = fq.fp8q_rmsnorm_quant(to_dev_bf16(x), to_dev_bf16(w[None, :])[0], 1e-6, H)
    y = fq.fp8q_scaled_mm(qa, to_dev_codes(b), sa.reshape(-1), torch.from_numpy(sb.reshape(-1)).cuda())
    torch.cuda.synchronize()
    a_ref, sa_ref = oracle.rmsnorm_quant(x, w, 1e-6, H)
    y_ref, ad = oracle.scaled_mm(a_ref, b, sa_ref.reshape(-1), sb.reshape(-1))
    gemm_tolerance_check(bf16_to_np(y), y_ref, ad, "tiny chain")
