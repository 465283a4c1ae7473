"""Decode-sized GEMMs (M <= 8 tokens) on the warp-MMA weight-streaming
variant (swap_ab = 1, split_k = 1, block_n = 8) against the oracle.

Shapes cover K with fewer 128-deep blocks than the kernel's warps, ragged
N (a multiple of 16, not of 128, for per-token scales), every M from 1 to 8,
per-tensor scales, outputs written into a larger buffer (nothing outside
[M, N] may change) and bit-identical reruns.  The Qwen3-32B decode shapes run
on the automatic variant in tests/test_gpu_gemm.py.
"""
import numpy as np
import pytest
import torch

import fp8q_inputs as inp
import oracle
from helpers import bf16_to_np, gemm_tolerance_check, to_dev_codes

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import fp8_quantized_linear_rms_b200 as fq   # fails loudly if libfp8q.so is missing

DECODE = (1, 1, 8)     # swap_ab, split_k, block_n


@pytest.fixture(autouse=True)
def _decode_variant():
    fq.fp8q_force_gemm_variant(*DECODE)
    yield
    fq.fp8q_force_gemm_variant()
    assert fq.fp8q_last_device_status() == fq.OK


def _pt(a, b, sa, sb, y=None):
    out = fq.fp8q_scaled_mm(to_dev_codes(a), to_dev_codes(b), torch.from_numpy(sa).cuda(),
                            torch.from_numpy(sb).cuda(), y=y)
    torch.cuda.synchronize()
    return out


def _bw(a, b, sa, sb, layout="row_major", y=None):
    sa_d = torch.from_numpy(np.ascontiguousarray(sa.T if layout == "group_major" else sa)).cuda()
    out = fq.fp8q_scaled_mm_blockwise(to_dev_codes(a), to_dev_codes(b), sa_d, torch.from_numpy(sb).cuda(),
                                      a_scale_layout=layout, y=y)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("M", [1, 2, 3, 5, 8])
@pytest.mark.parametrize("N,K", [(16, 128), (272, 384), (512, 1024), (128, 2304)])
def test_decode_per_token(M, N, K):
    a = inp.random_e4m3_codes(9000 + M * 31 + K, (M, K))
    b = inp.random_e4m3_codes(9100 + N + K, (N, K))
    sa = inp.random_scales(9200 + M, (M,))
    sb = inp.random_scales(9300 + N, (N,))
    y = bf16_to_np(_pt(a, b, sa, sb))
    y_ref, ad = oracle.scaled_mm(a, b, sa, sb)
    gemm_tolerance_check(y, y_ref, ad, f"decode per-token M={M} N={N} K={K}")


@pytest.mark.parametrize("layout", ["row_major", "group_major"])
@pytest.mark.parametrize("M", [1, 2, 4, 7, 8])
@pytest.mark.parametrize("N,K", [(128, 128), (384, 640), (256, 2048)])
def test_decode_blockwise(M, N, K, layout):
    a = inp.random_e4m3_codes(9400 + M * 17 + K, (M, K))
    b = inp.random_e4m3_codes(9500 + N + K, (N, K))
    sa = inp.random_scales(9600 + M, (M, K // 128))
    sb = inp.random_scales(9700 + N, (N // 128, K // 128))
    y = bf16_to_np(_bw(a, b, sa, sb, layout))
    y_ref, ad = oracle.scaled_mm_blockwise(a, b, sa, sb)
    gemm_tolerance_check(y, y_ref, ad, f"decode blockwise M={M} N={N} K={K} {layout}")


@pytest.mark.parametrize("per_token,per_channel", [(False, False), (False, True), (True, False)])
def test_decode_per_tensor_scales(per_token, per_channel):
    M, N, K = 6, 256, 512
    a = inp.random_e4m3_codes(9800, (M, K))
    b = inp.random_e4m3_codes(9801, (N, K))
    sa = inp.random_scales(9802, (M if per_token else 1,))
    sb = inp.random_scales(9803, (N if per_channel else 1,))
    y = bf16_to_np(_pt(a, b, sa, sb))
    y_ref, ad = oracle.scaled_mm(a, b, sa, sb)
    gemm_tolerance_check(y, y_ref, ad, "decode per-tensor scales")


@pytest.mark.parametrize("blockwise", [False, True])
def test_decode_canaries_and_determinism(blockwise):
    M, N, K = 5, 384, 1024
    a = inp.random_e4m3_codes(9900, (M, K))
    b = inp.random_e4m3_codes(9901, (N, K))
    sa = inp.random_scales(9902, (M, K // 128) if blockwise else (M,))
    sb = inp.random_scales(9903, (N // 128, K // 128) if blockwise else (N,))
    big = torch.full((M + 3, N + 24), 7.0, dtype=torch.bfloat16, device="cuda")
    y = big[:M, :N]
    outs = []
    for _ in range(3):
        (_bw if blockwise else _pt)(a, b, sa, sb, y=y)
        outs.append(y.clone())
    for o in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16))
    full = big.float().cpu().numpy()
    assert np.all(full[:, N:] == 7.0) and np.all(full[M:, :] == 7.0)
    y_ref, ad = (oracle.scaled_mm_blockwise if blockwise else oracle.scaled_mm)(a, b, sa, sb)
    gemm_tolerance_check(bf16_to_np(y), y_ref, ad, "decode canary case")


def test_decode_variant_rejects_more_than_eight_tokens():
    M, N, K = 9, 128, 256
    a = inp.random_e4m3_codes(9950, (M, K))
    b = inp.random_e4m3_codes(9951, (N, K))
    with pytest.raises(fq.Fp8qError) as e:
        _pt(a, b, inp.random_scales(9952, (M,)), inp.random_scales(9953, (N,)))
    assert e.value.status == fq.ERR_UNSUPPORTED
