"""GPU parity of the gate_up GEMM with the SiLU*mul 1x128 quant fused into its
epilogue (fp8q_scaled_mm_blockwise_silu_quant).

Exact mode: the fused op must give exactly what the chain it replaces gives:
the blockwise GEMM run with the same 128x256 whole-K variant (bf16 h =
[gate | up]) followed by fp8q_silu_mul_quant(h, 128) -- codes and scales
bit-identical -- and the oracle's SiLU*mul quant of that h (codes and scales
bit-identical).  Fast mode (the default): scales bit-identical to the
oracle's, codes within the fused-quant tolerance (>= 99.9% identical, the
rest one step away).  Against the oracle's own fp64 GEMM the chain meets the
GEMM tolerance, which the blockwise GEMM tests check.
"""
import numpy as np
import pytest
import torch

import fp8q_inputs as inp
import oracle
from helpers import (assert_fused_quant_close, codes_np, config_rows, fused_quant_exact, quantized_weights,
                     to_dev_codes)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _exact_standalone_quant():
    # the fused epilogue computes y exactly; the standalone op it is compared
    # with bit for bit runs in its exact mode
    with fused_quant_exact(True):
        yield

if torch.cuda.is_available():
    import fp8_quantized_linear_rms_b200 as fq   # fails loudly if libfp8q.so is missing


@pytest.fixture(autouse=True)
def _auto_variant():
    yield
    if torch.cuda.is_available():
        fq.fp8q_force_gemm_variant()
        assert fq.fp8q_last_device_status() == fq.OK


def _deinterleave(hi: torch.Tensor) -> torch.Tensor:
    """bf16 [M, 2I] with 128-column blocks [g0 | u0 | g1 | u1 ...] -> [gate | up]."""
    M, N2 = hi.shape
    nb = N2 // 256
    v = hi.reshape(M, nb, 2, 128)
    return torch.cat([v[:, :, 0].reshape(M, -1), v[:, :, 1].reshape(M, -1)], dim=1).contiguous()


def _run(a, sa, b, sb, layout, ue8m0, rows=None):
    """(fused q, fused s, chain q, chain s, h) on the device; h de-interleaved."""
    M, K = a.shape
    ad = to_dev_codes(a)
    sad = torch.from_numpy(np.ascontiguousarray(sa.T if layout == "group_major" else sa)).cuda()
    bi = fq.interleave_gate_up(to_dev_codes(b).view(torch.uint8)).view(torch.float8_e4m3fn)
    sbi = fq.interleave_gate_up(torch.from_numpy(sb).cuda(), block=1)
    q, s = fq.fp8q_scaled_mm_blockwise_silu_quant(ad, bi, sad, sbi, a_scale_layout=layout, ue8m0=ue8m0)
    fq.fp8q_force_gemm_variant(0, 1, 256, 0)
    hi = fq.fp8q_scaled_mm_blockwise(ad, bi, sad, sbi, a_scale_layout=layout)
    fq.fp8q_force_gemm_variant()
    h = _deinterleave(hi)
    q2, s2 = fq.fp8q_silu_mul_quant(h, 128, ue8m0)
    torch.cuda.synchronize()
    return q, s, q2, s2, h


@pytest.mark.parametrize("ue8m0", [False, True, "packed"])
@pytest.mark.parametrize("layout", ["row_major", "group_major"])
@pytest.mark.parametrize("M,I,K", [(1, 256, 256), (100, 384, 512), (300, 640, 1024)])
def test_fused_gate_up_silu_quant_equals_the_chain(M, I, K, layout, ue8m0):
    a = inp.random_e4m3_codes(M * 3 + K, (M, K))
    b = inp.random_e4m3_codes(I * 5 + K, (2 * I, K))
    sa = inp.random_scales(M + 11, (M, K // 128))
    sb = inp.random_scales(I + 12, (2 * I // 128, K // 128))
    q, s, q2, s2, h = _run(a, sa, b, sb, layout, ue8m0)
    assert torch.equal(q.view(torch.uint8), q2.view(torch.uint8))
    assert torch.equal(s, s2)
    hb = h.view(torch.int16).cpu().numpy().view(np.uint16)
    q_ref, s_ref = oracle.silu_mul_quant(hb, 128, ue8m0)
    np.testing.assert_array_equal(codes_np(q), q_ref)
    np.testing.assert_array_equal(s.cpu().numpy(), s_ref)          # output scales row-major [M, I/128]


@pytest.mark.parametrize("model,M", [("8b", 2048), ("32b", 8192)])
def test_fused_gate_up_silu_quant_config(model, M):
    # Qwen3 gate_up with heavy-tailed activations quantized by the oracle and
    # N(0, 0.02) weights in 128x128 blocks; all rows against the chain on the
    # GPU, sampled rows against the oracle's quant of the chain's h
    shapes = inp.linear_shapes(inp.QWEN3_8B if model == "8b" else inp.QWEN3_32B)
    K, N2 = shapes["gate_up"]
    x = inp.heavy_tailed_bf16(1300 + M, M, K)
    a, sa = oracle.group_quant(x, 128)
    b, sb = quantized_weights(N2 * 7 + K, N2, K, True)
    q, s, q2, s2, h = _run(a, sa, b, sb, "group_major", False)
    assert torch.equal(q.view(torch.uint8), q2.view(torch.uint8))
    assert torch.equal(s, s2)
    rows = config_rows(M, 1400 + M)
    hb = h[torch.from_numpy(rows).cuda()].view(torch.int16).cpu().numpy().view(np.uint16)
    q_ref, s_ref = oracle.silu_mul_quant(hb, 128)
    np.testing.assert_array_equal(codes_np(q)[rows], q_ref)
    np.testing.assert_array_equal(s.cpu().numpy()[rows], s_ref)


def _fast_vs_oracle(a, sa, b, sb, layout, ue8m0, what, rows=None):
    with fused_quant_exact(False):
        q, s, _, _, h = _run(a, sa, b, sb, layout, ue8m0)
    if rows is None:
        rows = np.arange(a.shape[0])
    hb = h[torch.from_numpy(rows).cuda()].view(torch.int16).cpu().numpy().view(np.uint16)
    q_ref, s_ref = oracle.silu_mul_quant(hb, 128, ue8m0)
    sg = s.cpu().numpy()[rows]                        # output scales row-major [M, I/128]
    np.testing.assert_array_equal(sg, s_ref)
    n = assert_fused_quant_close(codes_np(q)[rows], sg, q_ref, s_ref, what)
    print(f"{what}: {n} of {q_ref.size} codes differ")


@pytest.mark.parametrize("ue8m0", [False, "packed"])
@pytest.mark.parametrize("M,I,K", [(1, 256, 256), (100, 384, 512), (300, 640, 1024)])
def test_fused_gate_up_silu_quant_fast_mode(M, I, K, ue8m0):
    # random codes and scales: gates of every magnitude and sign (exact
    # products at large gates, gates below -85, tiny values), the routes the
    # fast epilogue must still take exactly
    a = inp.random_e4m3_codes(M * 3 + K + 1, (M, K))
    b = inp.random_e4m3_codes(I * 5 + K + 1, (2 * I, K))
    sa = inp.random_scales(M + 21, (M, K // 128))
    sb = inp.random_scales(I + 22, (2 * I // 128, K // 128))
    _fast_vs_oracle(a, sa, b, sb, "group_major", ue8m0, f"fused fast M={M} I={I} K={K} {ue8m0}")


@pytest.mark.parametrize("model,M", [("8b", 512), ("32b", 2048)])
def test_fused_gate_up_silu_quant_fast_mode_config(model, M):
    shapes = inp.linear_shapes(inp.QWEN3_8B if model == "8b" else inp.QWEN3_32B)
    K, N2 = shapes["gate_up"]
    x = inp.heavy_tailed_bf16(1500 + M, M, K)
    a, sa = oracle.group_quant(x, 128)
    b, sb = quantized_weights(N2 * 7 + K + 1, N2, K, True)
    _fast_vs_oracle(a, sa, b, sb, "group_major", False, f"fused fast {model} M={M}",
                    rows=config_rows(M, 1600 + M))
