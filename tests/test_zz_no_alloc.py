"""fp8q_scaled_mm_blockwise_noalloc, the GEMM entry point for callers that
cannot allocate device memory (an engine that pre-reserved all free HBM, a
plugin that is handed only its inputs and outputs, a path where cudaMalloc's
possible device synchronization is not allowed).  It runs the blockwise GEMM
with the library's fixed 16 MiB scratch array instead of a caller workspace.

Called through the C ABI, on split-K shapes (so the scratch is really used),
twice in a row per shape: both calls must agree with the workspace entry point
fp8q_scaled_mm_blockwise within the GEMM tolerance of the other tests
(|y - y_ref| <= 2^-8 |y_ref| + 1e-3 sum_k |a_k b_k|).  This file is collected
last on purpose, and passes alone in a fresh process as well.
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


@pytest.mark.parametrize("M,N,K", [(16, 5120, 25600), (8, 5120, 8192), (1, 5120, 25600), (64, 4096, 12288)])
def test_noalloc_matches_workspace_entry_point(M, N, K):
    fq.fp8q_force_gemm_variant()
    v = fq.fp8q_select_gemm_variant(M, N, K, True)
    assert v["split_k"] != 1, "the shape must exercise the split-K / stream-K scratch"
    assert 0 < fq.fp8q_workspace_bytes(M, N, K, True) <= fq.NOALLOC_SCRATCH_BYTES
    _compare_two_calls(M, N, K)


# (N, K) of the Qwen3-8B / Qwen3-32B linear layers and the M searched for a
# shape whose automatic variant needs more scratch than the fixed array
_LAYERS = [(6144, 4096), (4096, 4096), (24576, 4096), (4096, 12288), (10240, 5120),
           (5120, 8192), (51200, 5120), (5120, 25600)]
_MS = [1, 16, 32, 64, 128, 256, 384, 512, 1024]


def test_noalloc_runs_whole_k_tiles_when_the_split_scratch_does_not_fit():
    # the automatic variant of the chosen shape wants more split-K / stream-K
    # scratch than the fixed array holds: the call runs the same tiles with
    # whole K ranges.  Which shapes do depends on the measured variant table,
    # so the smallest such shape is looked up.
    fq.fp8q_force_gemm_variant()
    big = [(M * N * K, M, N, K) for N, K in _LAYERS for M in _MS
           if fq.fp8q_workspace_bytes(M, N, K, True) > fq.NOALLOC_SCRATCH_BYTES]
    if not big:
        pytest.skip("no layer shape's automatic variant outgrows the fixed scratch array")
    _, M, N, K = min(big)
    _compare_two_calls(M, N, K)


def _compare_two_calls(M, N, K):
    a = to_dev_codes(inp.random_e4m3_codes(M + 1, (M, K)))
    b = to_dev_codes(inp.random_e4m3_codes(N + 2, (N, K)))
    sa = torch.from_numpy(inp.random_scales(3, (M, K // 128))).cuda()
    sb = torch.from_numpy(inp.random_scales(4, (N // 128, K // 128))).cuda()
    y_ws = fq.fp8q_scaled_mm_blockwise(a, b, sa, sb, workspace=fq.make_workspace(M, N, K, True))
    torch.cuda.synchronize()
    # the oracle's fp64 result and |a_k b_k| sums, on every row
    ref, absdot = oracle.scaled_mm_blockwise(a.view(torch.uint8).cpu().numpy(),
                                             b.view(torch.uint8).cpu().numpy(),
                                             sa.cpu().numpy(), sb.cpu().numpy())
    y_ws_np = bf16_to_np(y_ws)
    gemm_tolerance_check(y_ws_np, ref, absdot, "workspace entry point")
    # the same variant sums in the same order: bit-identical to the workspace entry
    v = fq.fp8q_select_gemm_variant(M, N, K, True)
    same_variant = fq.fp8q_workspace_bytes(M, N, K, True) <= fq.NOALLOC_SCRATCH_BYTES
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        st = fq.lib.fp8q_scaled_mm_blockwise_noalloc(a.data_ptr(), b.data_ptr(), sa.data_ptr(),
                                                     K // 128, 1, sb.data_ptr(), M, N, K,
                                                     y.data_ptr(), N, stream)
        assert st == fq.OK, fq.fp8q_status_string(st)
        torch.cuda.synchronize()
        assert fq.fp8q_last_device_status() == fq.OK
        got = bf16_to_np(y)
        gemm_tolerance_check(got, ref, absdot, f"noalloc call {call + 1} ({v})")
        if same_variant:
            assert np.array_equal(got, y_ws_np), \
                f"noalloc call {call + 1} differs from the workspace entry point"


def test_noalloc_rejects_shapes_beyond_its_scratch():
    M, N, K = 256, 4096, 12288
    fq.fp8q_force_gemm_variant(0, 16, 256)      # 16 x 32 tiles x 16 splits of 128x256 fp32
    try:
        assert fq.fp8q_workspace_bytes(M, N, K, True) > fq.NOALLOC_SCRATCH_BYTES
        a = torch.zeros((M, K), dtype=torch.uint8, device="cuda")
        b = torch.zeros((N, K), dtype=torch.uint8, device="cuda")
        s = torch.ones(N * K // 128, dtype=torch.float32, device="cuda")
        y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        st = fq.lib.fp8q_scaled_mm_blockwise_noalloc(a.data_ptr(), b.data_ptr(), s.data_ptr(),
                                                     K // 128, 1, s.data_ptr(), M, N, K,
                                                     y.data_ptr(), N, None)
        assert st == fq.ERR_UNSUPPORTED
    finally:
        fq.fp8q_force_gemm_variant()
