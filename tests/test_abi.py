"""The C-ABI library: it loads, exports every function include/fp8q.h declares,
and validates arguments on the host (no kernel is launched by these calls, so
they run without a GPU)."""
import ctypes
import os
import re

import pytest

import fp8_quantized_linear_rms_b200 as fq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_library_exports_every_declared_function():
    names = fq.header_functions()
    assert len(names) == 22
    for n in names:
        assert hasattr(fq.lib, n), n
        assert callable(getattr(fq, n)), f"binding lacks {n}"


def test_fused_quant_mode_switch():
    # host-side setting only: no GPU needed
    assert fq.fp8q_get_fused_quant_exact() is False          # default: fast y, exact scales
    try:
        fq.fp8q_set_fused_quant_exact(True)
        assert fq.fp8q_get_fused_quant_exact() is True
        assert fq.lib.fp8q_set_fused_quant_exact(2) == fq.ERR_INVALID_ARG
        assert fq.lib.fp8q_set_fused_quant_exact(-1) == fq.ERR_INVALID_ARG
        assert fq.fp8q_get_fused_quant_exact() is True        # unchanged by a rejected value
    finally:
        fq.fp8q_set_fused_quant_exact(False)
    assert fq.fp8q_get_fused_quant_exact() is False


def test_status_strings_and_version():
    assert fq.fp8q_version().startswith("fp8q")
    for s in range(5):
        assert fq.fp8q_status_string(s)
    assert fq.fp8q_status_string(99) == "unknown status"


def test_invalid_arguments_rejected_before_launch():
    L = fq.lib
    fake = 1 << 20   # a 16-byte-aligned address that is never dereferenced
    # null pointers with M > 0
    assert L.fp8q_group_quant(None, 4, 256, 256, 128, 0, fake, 256, fake, 2, 1, None) == fq.ERR_INVALID_ARG
    # group size not 128 or K; K not a multiple of 16; ldx too small; bad ue8m0
    assert L.fp8q_group_quant(fake, 4, 256, 256, 64, 0, fake, 256, fake, 2, 1, None) == fq.ERR_INVALID_ARG
    assert L.fp8q_group_quant(fake, 4, 200, 208, 200, 0, fake, 208, fake, 1, 1, None) == fq.ERR_INVALID_ARG
    assert L.fp8q_group_quant(fake, 4, 256, 128, 128, 0, fake, 256, fake, 2, 1, None) == fq.ERR_INVALID_ARG
    assert L.fp8q_group_quant(fake, 4, 256, 256, 128, 3, fake, 256, fake, 2, 1, None) == fq.ERR_INVALID_ARG
    # misaligned input
    assert L.fp8q_group_quant(fake + 2, 4, 256, 256, 128, 0, fake, 256, fake, 2, 1, None) == fq.ERR_INVALID_ARG
    # negative eps, silu ldx < 2I
    assert L.fp8q_rmsnorm_quant(fake, fake, ctypes.c_float(-1.0), 4, 256, 256, 128, 0, fake, 256, fake,
                                2, 1, None) == fq.ERR_INVALID_ARG
    assert L.fp8q_silu_mul_quant(fake, 4, 256, 256, 128, 0, fake, 256, fake, 2, 1, None) == fq.ERR_INVALID_ARG
    # GEMMs: N % 16, K % 16, ldy < N, blockwise K % 128 and N % 128
    assert L.fp8q_scaled_mm(fake, fake, fake, 1, fake, 1, 4, 24, 256, fake, 24, None, 0, None) == fq.ERR_INVALID_ARG
    assert L.fp8q_scaled_mm(fake, fake, fake, 1, fake, 1, 4, 32, 40, fake, 32, None, 0, None) == fq.ERR_INVALID_ARG
    assert L.fp8q_scaled_mm(fake, fake, fake, 1, fake, 1, 4, 32, 256, fake, 16, None, 0, None) == fq.ERR_INVALID_ARG
    assert L.fp8q_scaled_mm_blockwise(fake, fake, fake, 2, 1, fake, 4, 128, 200, fake, 128, None, 0,
                                      None) == fq.ERR_INVALID_ARG
    assert L.fp8q_scaled_mm_blockwise(fake, fake, fake, 2, 1, fake, 4, 192, 256, fake, 192, None, 0,
                                      None) == fq.ERR_INVALID_ARG
    # activation-scale strides whose offsets leave the 32-bit range
    assert L.fp8q_scaled_mm_blockwise(fake, fake, fake, 1 << 30, 1, fake, 4, 128, 256, fake, 128, None,
                                      0, None) == fq.ERR_INVALID_ARG
    assert L.fp8q_scaled_mm_blockwise_noalloc(fake, fake, fake, 1, 1 << 29, fake, 4, 128, 256, fake,
                                              128, None) == fq.ERR_INVALID_ARG
    # E8M0 GEMM: N or K not a multiple of 128, null scale bytes, misaligned y
    e8 = L.fp8q_scaled_mm_blockwise_e8m0
    assert e8(fake, fake, fake, 2, 1, fake, 4, 192, 256, fake, 192, None, 0, None) == fq.ERR_INVALID_ARG
    assert e8(fake, fake, fake, 2, 1, fake, 4, 128, 200, fake, 128, None, 0, None) == fq.ERR_INVALID_ARG
    assert e8(fake, fake, None, 2, 1, fake, 4, 128, 256, fake, 128, None, 0, None) == fq.ERR_INVALID_ARG
    assert e8(fake, fake, fake, 2, 1, fake, 4, 128, 256, fake + 8, 128, None, 0, None) == fq.ERR_INVALID_ARG
    # residual add: residual leading dimension below H, null residual
    ar = L.fp8q_add_rmsnorm_quant
    assert ar(fake, fake, fake, ctypes.c_float(1e-6), 4, 256, 256, 128, 128, 0, fake, 256, fake, 2, 1,
              None) == fq.ERR_INVALID_ARG
    assert ar(fake, None, fake, ctypes.c_float(1e-6), 4, 256, 256, 256, 128, 0, fake, 256, fake, 2, 1,
              None) == fq.ERR_INVALID_ARG
    assert ar(None, None, None, ctypes.c_float(1e-6), 0, 256, 256, 256, 128, 0, None, 256, None, 2, 1,
              None) == fq.OK
    # qk norm + rope: unsupported head size, ld too small, bad is_neox, zero tokens
    qr = L.fp8q_qk_norm_rope
    assert qr(fake, 4, 1280, 8, 1, 1, 96, ctypes.c_float(1e-6), fake, fake, fake, 16, fake, 1,
              None) == fq.ERR_UNSUPPORTED
    assert qr(fake, 4, 1000, 8, 1, 1, 128, ctypes.c_float(1e-6), fake, fake, fake, 16, fake, 1,
              None) == fq.ERR_INVALID_ARG
    assert qr(fake, 4, 1280, 8, 1, 1, 128, ctypes.c_float(1e-6), fake, fake, fake, 16, fake, 2,
              None) == fq.ERR_INVALID_ARG
    assert qr(None, 0, 1280, 8, 1, 1, 128, ctypes.c_float(1e-6), None, None, None, 16, None, 1,
              None) == fq.OK
    # fused gate_up + SiLU quant: 2I not a multiple of 256, ldq < I, bad ue8m0
    fs = L.fp8q_scaled_mm_blockwise_silu_quant
    assert fs(fake, fake, fake, 2, 1, fake, 4, 384, 256, 0, fake, 192, fake, 2, 1, None) == fq.ERR_INVALID_ARG
    assert fs(fake, fake, fake, 2, 1, fake, 4, 512, 256, 0, fake, 128, fake, 2, 1, None) == fq.ERR_INVALID_ARG
    assert fs(fake, fake, fake, 2, 1, fake, 4, 512, 256, 3, fake, 256, fake, 2, 1, None) == fq.ERR_INVALID_ARG
    assert fs(None, None, None, 2, 1, None, 0, 512, 256, 0, None, 256, None, 2, 1, None) == fq.OK
    # int8: K beyond the exact-sum range, group size, null scales
    assert L.fp8q_scaled_mm_i8(fake, fake, fake, 1, fake, 1, 4, 128, 133152 + 16, fake, 128, None, 0,
                               None) == fq.ERR_INVALID_ARG
    assert L.fp8q_group_quant_i8(fake, 4, 256, 256, 64, fake, 256, fake, 2, 1, None) == fq.ERR_INVALID_ARG
    assert L.fp8q_rmsnorm_quant_i8(fake, fake, ctypes.c_float(1e-6), 4, 256, 256, 128, fake, 256, None,
                                   2, 1, None) == fq.ERR_INVALID_ARG
    assert L.fp8q_silu_mul_quant_i8(fake, 4, 256, 256, 128, fake, 256, fake, 2, 1, None) == fq.ERR_INVALID_ARG
    # packed E8M0 quant scales need no alignment; ue8m0 beyond 2 is rejected
    assert L.fp8q_group_quant(fake, 4, 256, 256, 128, 3, fake, 256, fake + 1, 2, 1, None) == fq.ERR_INVALID_ARG
    assert L.fp8q_group_quant(fake, 4, 256, 256, 128, 1, fake, 256, fake + 1, 2, 1, None) == fq.ERR_INVALID_ARG


def test_zero_rows_is_a_noop_without_pointers():
    L = fq.lib
    assert L.fp8q_group_quant(None, 0, 256, 256, 128, 0, None, 256, None, 2, 1, None) == fq.OK
    assert L.fp8q_scaled_mm(None, None, None, 1, None, 1, 0, 256, 256, None, 256, None, 0, None) == fq.OK
    assert L.fp8q_scaled_mm_blockwise(None, None, None, 2, 1, None, 0, 256, 256, None, 256, None, 0,
                                      None) == fq.OK
    assert L.fp8q_scaled_mm_blockwise_e8m0(None, None, None, 2, 1, None, 0, 256, 256, None, 256, None,
                                           0, None) == fq.OK


def _variant_table():
    """Rows of the compiled-in variant table, read from its source text."""
    path = os.path.join(ROOT, "fp8_quantized_linear_rms_b200", "csrc", "fp8q_variant_table.inc")
    rows = []
    for line in open(path):
        m = re.match(r"\{(-?\d+), (\d+), (\d+), (\d+), (\d+), (\d+), (\d+), (\d+)\},", line)
        if m:
            rows.append(tuple(int(x) for x in m.groups()))
    return rows


def test_variant_table_lookup():
    rows = _variant_table()
    assert len(rows) >= 100
    keys = {}
    for bw, m_max, n, k, swap, split, bn, pair in rows:
        keys.setdefault((bw, n, k), []).append(m_max)
        want = {"swap_ab": swap, "split_k": split, "block_n": bn, "cta_pair": pair}
        assert fq.fp8q_select_gemm_variant(m_max, n, k, bool(bw)) == want
    # an M between buckets takes the next larger bucket; above all, the largest
    for (bw, n, k), ms in keys.items():
        ms = sorted(ms)
        by_m = {r[1]: r for r in rows if (r[0], r[2], r[3]) == (bw, n, k)}
        for lo, hi in zip(ms, ms[1:]):
            if hi - lo > 1:
                r = by_m[hi]
                assert fq.fp8q_select_gemm_variant(lo + 1, n, k, bool(bw)) == \
                    {"swap_ab": r[4], "split_k": r[5], "block_n": r[6], "cta_pair": r[7]}
        r = by_m[ms[-1]]
        assert fq.fp8q_select_gemm_variant(ms[-1] * 4, n, k, bool(bw)) == \
            {"swap_ab": r[4], "split_k": r[5], "block_n": r[6], "cta_pair": r[7]}


def test_int8_and_e8m0_never_take_the_decode_variant():
    # the warp-MMA decode kernel serves fp8 with fp32 scales only; where the
    # per-token table picks it, the int8 and E8M0 schemes take Swap-AB tiles
    for M in (1, 2, 8):
        for N, K in ((10240, 5120), (6144, 4096), (3072, 2560)):
            assert fq.fp8q_select_gemm_variant(M, N, K, False)["block_n"] == 8
            for scheme in (2, 3):
                v = fq.fp8q_select_gemm_variant(M, N, K, scheme)
                assert v["block_n"] in (16, 32, 64, 128) and v["swap_ab"] == 1, (M, N, K, scheme, v)


def test_variant_selection_host_logic():
    # shapes outside the table: the warp-MMA decode variant for M <= 8 (K up to
    # 16384), Swap-AB with tokens padded to 16/32/64/128 for other small M, no
    # swap for large M
    N, K = 3072, 2560
    for M in (1, 5, 8):
        assert fq.fp8q_select_gemm_variant(M, N, K, True) == \
            {"swap_ab": 1, "split_k": 1, "block_n": 8, "cta_pair": 0}
        assert fq.fp8q_select_gemm_variant(M, N, K, False)["block_n"] == 8
    assert fq.fp8q_select_gemm_variant(1, N, 32768, True)["block_n"] == 16
    assert fq.fp8q_select_gemm_variant(9, N, K, True)["block_n"] == 16
    assert fq.fp8q_select_gemm_variant(33, N, K, True)["block_n"] == 64
    assert fq.fp8q_select_gemm_variant(100, N, K, False)["block_n"] == 128
    v = fq.fp8q_select_gemm_variant(8192, N, K, True)
    assert v == {"swap_ab": 0, "split_k": 1, "block_n": 256, "cta_pair": 0}
    # per-token scales, M >= 512 and at least 40 tiles of 256 x 256: CTA pairs
    v = fq.fp8q_select_gemm_variant(8192, N, K, False)
    assert v == {"swap_ab": 0, "split_k": 1, "block_n": 256, "cta_pair": 1}
    assert fq.fp8q_select_gemm_variant(512, 5120 - 128, K, False)["cta_pair"] == 1   # 2 x 20 tiles
    assert fq.fp8q_select_gemm_variant(512, 4096 + 128, K, False)["cta_pair"] == 0   # 2 x 17 tiles
    assert fq.fp8q_select_gemm_variant(256, 51200 + 128, K, False)["cta_pair"] == 0  # M < 512
    # 24 tiles: whole-K ranges split so that the tiles fill the SMs, each
    # range at least 8 K blocks; blockwise with M > 16 takes stream-K
    assert fq.fp8q_select_gemm_variant(16, N, K, False)["split_k"] == 2
    assert fq.fp8q_select_gemm_variant(16, N, 8 * 128 * 6, False)["split_k"] == 6
    assert fq.fp8q_select_gemm_variant(64, N, K, True)["split_k"] == 0
    assert fq.fp8q_workspace_bytes(64, N, K, True) > 0
    assert fq.fp8q_workspace_bytes(8192, 51200, 5120, False) == 0
    # forcing
    fq.fp8q_force_gemm_variant(0, 2, 256)
    assert fq.fp8q_select_gemm_variant(8192, 51200, 5120, False) == \
        {"swap_ab": 0, "split_k": 2, "block_n": 256, "cta_pair": 0}
    fq.fp8q_force_gemm_variant(0, 1, 128, cta_pair=1)
    assert fq.fp8q_select_gemm_variant(8192, 51200, 5120, True) == \
        {"swap_ab": 0, "split_k": 1, "block_n": 128, "cta_pair": 1}
    assert fq.fp8q_workspace_bytes(8192, 51200, 5120, True) == 0
    fq.fp8q_force_gemm_variant()
    with pytest.raises(fq.Fp8qError):
        fq.fp8q_force_gemm_variant(0, 1, 48)


def test_e8m0_variant_selection_host_logic():
    # The E8M0 GEMM follows the per-token scheme's choice, single CTAs only
    # (128x256 tiles where that scheme takes CTA pairs).
    for M, N, K in [(8192, 51200, 5120), (2048, 24576, 4096), (4096, 6144, 4096)]:
        v = fq.fp8q_select_gemm_variant(M, N, K, 2)
        pt = fq.fp8q_select_gemm_variant(M, N, K, False)
        assert v["cta_pair"] == 0 and v["swap_ab"] == 0 and v["block_n"] in (128, 256), v
        assert v["block_n"] == (256 if pt["cta_pair"] else pt["block_n"]), (v, pt)
    for M in (16, 32, 64):
        v = fq.fp8q_select_gemm_variant(M, 10240, 5120, 2)
        pt = fq.fp8q_select_gemm_variant(M, 10240, 5120, False)
        assert v == pt, (M, v, pt)
    assert fq.fp8q_workspace_bytes(8192, 51200, 5120, 2) == 0
    assert fq.fp8q_workspace_bytes(8192, 51200, 5120, 3) == 0
    # forcing: 224 is accepted (the E8M0 tile), an unsupported combination for
    # the scheme is reported by the GEMM call itself
    fq.fp8q_force_gemm_variant(0, 3, 224)
    assert fq.fp8q_select_gemm_variant(4096, 6144, 4096, 2) == \
        {"swap_ab": 0, "split_k": 3, "block_n": 224, "cta_pair": 0}
    assert fq.fp8q_workspace_bytes(4096, 6144, 4096, 2) > 0
    fq.fp8q_force_gemm_variant()


def test_interleave_gate_up_layout():
    import torch
    I, K = 256, 4
    w = torch.arange(2 * I * K, dtype=torch.float32).reshape(2 * I, K)
    wi = fq.interleave_gate_up(w)
    # block row 2j = gate rows [128 j, 128 j + 128), 2j + 1 = up rows [I + 128 j, ...)
    assert torch.equal(wi[0:128], w[0:128]) and torch.equal(wi[128:256], w[I:I + 128])
    assert torch.equal(wi[256:384], w[128:256]) and torch.equal(wi[384:512], w[I + 128:I + 256])
    s = torch.arange(2 * I // 128, dtype=torch.float32)[:, None].repeat(1, 3)
    si = fq.interleave_gate_up(s, block=1)
    assert si[:, 0].tolist() == [0.0, 2.0, 1.0, 3.0]
