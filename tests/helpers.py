"""Shared helpers of the GPU parity tests: move seeded inputs to the device,
compare against the oracle with the stated tolerances."""
from __future__ import annotations

import contextlib

import ml_dtypes
import numpy as np
import torch

import fp8q_inputs as inp


def to_dev_bf16(bits: np.ndarray, device="cuda", ld: int | None = None) -> torch.Tensor:
    """uint16 bf16 bits [M, L] -> bf16 CUDA tensor, optionally with a padded leading dim."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    if ld is None or ld == bits.shape[-1]:
        return t.to(device)
    M, L = bits.shape
    big = torch.full((M, ld), float("nan"), dtype=torch.bfloat16)
    big[:, :L] = t
    return big.to(device)[:, :L]


def to_dev_codes(codes: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).to(device)


def codes_np(q: torch.Tensor) -> np.ndarray:
    return q.contiguous().view(torch.uint8).cpu().numpy()


def e4m3_values(codes: np.ndarray) -> np.ndarray:
    return codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64)


def assert_fused_quant_close(q_gpu, s_gpu, q_ref, s_ref, what=""):
    """Tolerance for producer-fused quant: >= 99.9% of codes identical, the rest
    within one e4m3 step, scales within 1e-5 relative.  Returns the number of
    differing codes."""
    np.testing.assert_allclose(s_gpu, s_ref, rtol=1e-5, atol=0, err_msg=what)
    diff = q_gpu != q_ref
    n = int(diff.sum())
    assert n <= 1e-3 * q_ref.size, f"{what}: {n} of {q_ref.size} codes differ"
    if n:
        # one e4m3 step: neighbouring codes of the same sign (or +-0 / smallest subnormal)
        a = q_gpu[diff].astype(np.int32)
        b = q_ref[diff].astype(np.int32)
        same_sign = (a & 0x80) == (b & 0x80)
        step = np.abs((a & 0x7F) - (b & 0x7F)) <= 1
        zero_cross = ((a & 0x7F) <= 1) & ((b & 0x7F) <= 1)
        assert np.all((same_sign & step) | zero_cross), f"{what}: a code moved by more than one step"
    return n


def gemm_tolerance_check(y_gpu_bf16: np.ndarray, y_ref: np.ndarray, absdot: np.ndarray, what=""):
    """|y - y_ref| <= 2^-8 |y_ref| + 1e-3 sum_k |a_k b_k| (y_ref fp64, y from bf16)."""
    y = y_gpu_bf16.astype(np.float64)
    err = np.abs(y - y_ref)
    bound = 2.0 ** -8 * np.abs(y_ref) + 1e-3 * absdot
    bad = err > bound
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; first at "
                             f"{tuple(i)}: gpu {y[tuple(i)]} ref {y_ref[tuple(i)]} "
                             f"bound {bound[tuple(i)]}")


def bf16_to_np(y: torch.Tensor) -> np.ndarray:
    return y.float().cpu().numpy()


def sample_rows(M: int, n: int, seed: int) -> np.ndarray:
    """n seeded rows plus the first and last rows and the last partial 128-row tile."""
    g = np.random.default_rng(seed)
    rows = set(g.choice(M, size=min(n, M), replace=False).tolist())
    rows |= {0, M - 1}
    rows |= set(range(max(0, (M // 128) * 128), M))
    return np.array(sorted(rows), dtype=np.int64)


def config_rows(M: int, seed: int, n: int = 256, tile: int = 256) -> np.ndarray:
    """Rows for a config-size GEMM check (every column of each is compared):
    n seeded rows spread over every `tile`-row tile, half of each tile's share
    from its first 128 rows and half from its last 128 (the two CTAs of a
    256-row CTA-pair tile), plus every row of the last tile and the first and
    last rows.  M <= n: every row."""
    if M <= n:
        return np.arange(M, dtype=np.int64)
    g = np.random.default_rng(seed)
    ntiles = -(-M // tile)
    per = max(2, n // ntiles)
    rows = {0, M - 1}
    for t in range(ntiles):
        for lo, hi in ((t * tile, t * tile + tile // 2), (t * tile + tile // 2, (t + 1) * tile)):
            lo, hi = min(lo, M), min(hi, M)
            if hi > lo:
                rows |= set(g.choice(np.arange(lo, hi), size=min(per // 2, hi - lo), replace=False).tolist())
    rows |= set(range((ntiles - 1) * tile, M))
    return np.array(sorted(rows), dtype=np.int64)


def quantized_weights(seed: int, N: int, K: int, blockwise: bool):
    """Seeded W ~ N(0, 0.02) quantized by the ORACLE: per output channel
    (codes, s[N]) or in 128x128 blocks (codes, s[N/128, K/128])."""
    import oracle
    w = inp.weight_bf16(seed, N, K)
    if not blockwise:
        return oracle.group_quant(w, K)          # s [N, 1]
    # 128x128 blocks: amax over each block, codes per block scale
    wf = inp.bf16_bits_to_f32(w).reshape(N // 128, 128, K // 128, 128)
    amax = np.abs(wf).max(axis=(1, 3)).astype(np.float32)
    s = oracle.scale(amax)                                        # [N/128, K/128]
    t = (wf / s[:, None, :, None]).astype(np.float32)
    q = oracle.e4m3_encode(t).reshape(N, K)
    return q, s


@contextlib.contextmanager
def fused_quant_exact(exact=True):
    """Run the producer-fused quant ops in the given arithmetic mode (restored after)."""
    import fp8_quantized_linear_rms_b200 as fq
    prev = fq.fp8q_get_fused_quant_exact()
    fq.fp8q_set_fused_quant_exact(exact)
    try:
        yield
    finally:
        fq.fp8q_set_fused_quant_exact(prev)
