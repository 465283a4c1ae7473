"""Python binding of libfp8q, the B200 (sm_100a) FP8 W8A8 linear-layer path.

Argument marshalling only: every entry point takes torch CUDA tensors, checks
dtypes and shapes enough to pass the right pointers, and calls the C ABI of
``include/fp8q.h`` with the current CUDA stream.  All arithmetic runs in the
library's kernels; there is no CPU or PyTorch fallback, and importing this
package fails loudly if ``libfp8q.so`` is missing (build it with
``python fp8_quantized_linear_rms_b200/build.py``).

The names match the C ABI:
  fp8q_group_quant, fp8q_rmsnorm_quant, fp8q_add_rmsnorm_quant, fp8q_silu_mul_quant
                                                                (activation quant)
  fp8q_scaled_mm, fp8q_scaled_mm_blockwise, fp8q_scaled_mm_blockwise_e8m0,
  fp8q_scaled_mm_blockwise_silu_quant                           (scaled FP8 GEMMs)
  fp8q_workspace_bytes, fp8q_select_gemm_variant, fp8q_force_gemm_variant,
  fp8q_last_device_status, fp8q_status_string, fp8q_version
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libfp8q.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "fp8q.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libfp8q.so not found at {LIB_PATH}; build it with "
                      "`python fp8_quantized_linear_rms_b200/build.py`")

lib = ctypes.CDLL(LIB_PATH)

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT = range(5)

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_INT = ctypes.c_int


class GemmVariant(ctypes.Structure):
    """fp8q_gemm_variant: swap_ab, split_k, block_n, cta_pair."""
    _fields_ = [("swap_ab", ctypes.c_int), ("split_k", ctypes.c_int), ("block_n", ctypes.c_int),
                ("cta_pair", ctypes.c_int)]

    def as_dict(self):
        return {"swap_ab": self.swap_ab, "split_k": self.split_k, "block_n": self.block_n,
                "cta_pair": self.cta_pair}


_SIGS = {
    "fp8q_group_quant": (_INT, [_P, _I64, _I64, _I64, _INT, _INT, _P, _I64, _P, _I64, _I64, _P]),
    "fp8q_rmsnorm_quant": (_INT, [_P, _P, ctypes.c_float, _I64, _I64, _I64, _INT, _INT, _P, _I64,
                                  _P, _I64, _I64, _P]),
    "fp8q_silu_mul_quant": (_INT, [_P, _I64, _I64, _I64, _INT, _INT, _P, _I64, _P, _I64, _I64,
                                   _P]),
    "fp8q_add_rmsnorm_quant": (_INT, [_P, _P, _P, ctypes.c_float, _I64, _I64, _I64, _I64, _INT, _INT,
                                      _P, _I64, _P, _I64, _I64, _P]),
    "fp8q_set_fused_quant_exact": (_INT, [_INT]),
    "fp8q_get_fused_quant_exact": (_INT, []),
    "fp8q_scaled_mm": (_INT, [_P, _P, _P, _INT, _P, _INT, _I64, _I64, _I64, _P, _I64, _P,
                              ctypes.c_size_t, _P]),
    "fp8q_scaled_mm_blockwise": (_INT, [_P, _P, _P, _I64, _I64, _P, _I64, _I64, _I64, _P, _I64,
                                        _P, ctypes.c_size_t, _P]),
    "fp8q_scaled_mm_blockwise_silu_quant": (_INT, [_P, _P, _P, _I64, _I64, _P, _I64, _I64, _I64, _INT,
                                                   _P, _I64, _P, _I64, _I64, _P]),
    "fp8q_scaled_mm_blockwise_e8m0": (_INT, [_P, _P, _P, _I64, _I64, _P, _I64, _I64, _I64, _P,
                                             _I64, _P, ctypes.c_size_t, _P]),
    "fp8q_scaled_mm_blockwise_noalloc": (_INT, [_P, _P, _P, _I64, _I64, _P, _I64, _I64, _I64, _P,
                                                _I64, _P]),
    "fp8q_qk_norm_rope": (_INT, [_P, _I64, _I64, _INT, _INT, _INT, _INT, ctypes.c_float, _P, _P, _P,
                                 _I64, _P, _INT, _P]),
    "fp8q_group_quant_i8": (_INT, [_P, _I64, _I64, _I64, _INT, _P, _I64, _P, _I64, _I64, _P]),
    "fp8q_rmsnorm_quant_i8": (_INT, [_P, _P, ctypes.c_float, _I64, _I64, _I64, _INT, _P, _I64, _P,
                                     _I64, _I64, _P]),
    "fp8q_silu_mul_quant_i8": (_INT, [_P, _I64, _I64, _I64, _INT, _P, _I64, _P, _I64, _I64, _P]),
    "fp8q_scaled_mm_i8": (_INT, [_P, _P, _P, _INT, _P, _INT, _I64, _I64, _I64, _P, _I64, _P,
                                 ctypes.c_size_t, _P]),
    "fp8q_workspace_bytes": (ctypes.c_size_t, [_I64, _I64, _I64, _INT]),
    "fp8q_select_gemm_variant": (_INT, [_I64, _I64, _I64, _INT, ctypes.POINTER(GemmVariant)]),
    "fp8q_force_gemm_variant": (_INT, [ctypes.POINTER(GemmVariant)]),
    "fp8q_last_device_status": (_INT, [_P]),
    "fp8q_status_string": (ctypes.c_char_p, [_INT]),
    "fp8q_version": (ctypes.c_char_p, []),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(lib, _name)
    _f.restype = _res
    _f.argtypes = _args


class Fp8qError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {lib.fp8q_status_string(status).decode()} ({status})")


def header_functions() -> list[str]:
    """Names of every function include/fp8q.h declares."""
    with open(HEADER_PATH) as f:
        text = f.read()
    return re.findall(r"^FP8Q_API\s+[\w\s\*]+?\b(fp8q_\w+)\s*\(", text, flags=re.M)


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(fn: str, status: int) -> None:
    if status != OK:
        raise Fp8qError(fn, status)


def _need(t: torch.Tensor, dtype, name: str) -> None:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


def _rowmajor(t: torch.Tensor, name: str) -> int:
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError(f"{name} must be 2-D with unit column stride")
    return t.stride(0)


def _ue8m0_mode(ue8m0) -> int:
    """False / True / "packed" -> the ABI's 0 (fp32) / 1 (power-of-two fp32) / 2 (E8M0 bytes)."""
    if ue8m0 == "packed":
        return 2
    if ue8m0 in (False, True, 0, 1):
        return int(ue8m0)
    raise ValueError(f"ue8m0 must be False, True or 'packed', got {ue8m0!r}")


def _scales_out(M, L, group, layout, device, scales, mode=0):
    G = L // group if group > 0 and L % group == 0 else 0
    dt = torch.uint8 if mode == 2 else torch.float32
    if scales is None:
        if layout == "group_major":
            scales = torch.empty((G, M), dtype=dt, device=device)
        else:
            scales = torch.empty((M, G), dtype=dt, device=device)
    elif scales.dtype != dt:
        raise TypeError(f"scales must be {dt} for ue8m0 mode {mode}")
    if layout == "group_major":
        return scales, 1, M
    return scales, G, 1


# --------------------------------------------------------------- activation quant
def fp8q_group_quant(x: torch.Tensor, group_size: int, ue8m0: bool = False, q=None, scales=None,
                     scale_layout: str = "row_major", stream=None):
    """per_token_group_fp8_quant (group_size=128) / per-token quant (group_size=K).

    x: bf16 [M, K].  Returns (q float8_e4m3fn [M, K], scales fp32 [M, K/g]
    (row_major) or [K/g, M] (group_major)).  ue8m0: False, True (power-of-two
    fp32 scales) or "packed" (the same scales as uint8 E8M0 bytes).
    """
    _need(x, torch.bfloat16, "x")
    ldx = _rowmajor(x, "x")
    M, K = x.shape
    mode = _ue8m0_mode(ue8m0)
    if q is None:
        q = torch.empty((M, K), dtype=torch.float8_e4m3fn, device=x.device)
    scales, ssm, ssg = _scales_out(M, K, group_size, scale_layout, x.device, scales, mode)
    st = lib.fp8q_group_quant(x.data_ptr(), M, K, ldx, group_size, mode, q.data_ptr(),
                              _rowmajor(q, "q"), scales.data_ptr(), ssm, ssg, _stream(stream))
    _check("fp8q_group_quant", st)
    return q, scales


def fp8q_rmsnorm_quant(x: torch.Tensor, w: torch.Tensor, eps: float, group_size: int,
                       ue8m0: bool = False, q=None, scales=None, scale_layout: str = "row_major",
                       stream=None):
    """rms_norm_dynamic_per_token_quant (group_size=H) / rms_norm_per_block_quant (128)."""
    _need(x, torch.bfloat16, "x")
    _need(w, torch.bfloat16, "w")
    ldx = _rowmajor(x, "x")
    M, H = x.shape
    mode = _ue8m0_mode(ue8m0)
    if q is None:
        q = torch.empty((M, H), dtype=torch.float8_e4m3fn, device=x.device)
    scales, ssm, ssg = _scales_out(M, H, group_size, scale_layout, x.device, scales, mode)
    st = lib.fp8q_rmsnorm_quant(x.data_ptr(), w.data_ptr(), ctypes.c_float(eps), M, H, ldx,
                                group_size, mode, q.data_ptr(), _rowmajor(q, "q"),
                                scales.data_ptr(), ssm, ssg, _stream(stream))
    _check("fp8q_rmsnorm_quant", st)
    return q, scales


def fp8q_add_rmsnorm_quant(x: torch.Tensor, residual: torch.Tensor, w: torch.Tensor, eps: float,
                           group_size: int, ue8m0=False, q=None, scales=None,
                           scale_layout: str = "row_major", stream=None):
    """Residual add + RMSNorm quant: residual <- bf16(x + residual) in place, then
    rms_norm quant of the new residual.  Returns (q, scales)."""
    _need(x, torch.bfloat16, "x")
    _need(residual, torch.bfloat16, "residual")
    _need(w, torch.bfloat16, "w")
    ldx = _rowmajor(x, "x")
    ldr = _rowmajor(residual, "residual")
    M, H = x.shape
    if tuple(residual.shape) != (M, H):
        raise ValueError("residual must have x's shape")
    mode = _ue8m0_mode(ue8m0)
    if q is None:
        q = torch.empty((M, H), dtype=torch.float8_e4m3fn, device=x.device)
    scales, ssm, ssg = _scales_out(M, H, group_size, scale_layout, x.device, scales, mode)
    st = lib.fp8q_add_rmsnorm_quant(x.data_ptr(), residual.data_ptr(), w.data_ptr(), ctypes.c_float(eps),
                                    M, H, ldx, ldr, group_size, mode, q.data_ptr(), _rowmajor(q, "q"),
                                    scales.data_ptr(), ssm, ssg, _stream(stream))
    _check("fp8q_add_rmsnorm_quant", st)
    return q, scales


def fp8q_silu_mul_quant(x: torch.Tensor, group_size: int, ue8m0: bool = False, q=None,
                        scales=None, scale_layout: str = "row_major", stream=None):
    """silu_and_mul_dynamic_per_token_quant (group_size=I) / silu_and_mul_per_block_quant (128).

    x: bf16 [M, 2I] = [gate | up].
    """
    _need(x, torch.bfloat16, "x")
    ldx = _rowmajor(x, "x")
    M, I2 = x.shape
    I = I2 // 2
    mode = _ue8m0_mode(ue8m0)
    if q is None:
        q = torch.empty((M, I), dtype=torch.float8_e4m3fn, device=x.device)
    scales, ssm, ssg = _scales_out(M, I, group_size, scale_layout, x.device, scales, mode)
    st = lib.fp8q_silu_mul_quant(x.data_ptr(), M, I, ldx, group_size, mode, q.data_ptr(),
                                 _rowmajor(q, "q"), scales.data_ptr(), ssm, ssg, _stream(stream))
    _check("fp8q_silu_mul_quant", st)
    return q, scales


# --------------------------------------------------------------------- GEMMs
def fp8q_workspace_bytes(M: int, N: int, K: int, blockwise) -> int:
    """blockwise: False (scaled_mm), True (scaled_mm_blockwise) or 2 (the E8M0 GEMM)."""
    return int(lib.fp8q_workspace_bytes(M, N, K, int(blockwise)))


def make_workspace(M: int, N: int, K: int, blockwise, device="cuda") -> torch.Tensor | None:
    """A zero-filled workspace for a GEMM of this shape (None if it needs none)."""
    n = fp8q_workspace_bytes(M, N, K, blockwise)
    return torch.zeros(n, dtype=torch.uint8, device=device) if n else None


def _ws(ws, M, N, K, blockwise, device):
    """Pointer/size of the caller's workspace; when none is given and the shape
    needs one, a fresh zero-filled buffer (the C ABI itself never allocates)."""
    if ws is None:
        ws = make_workspace(M, N, K, blockwise, device)
    return (ws.data_ptr(), ws.numel() * ws.element_size(), ws) if ws is not None else (None, 0, None)


def fp8q_scaled_mm(a_q: torch.Tensor, b_q: torch.Tensor, a_scale: torch.Tensor,
                   b_scale: torch.Tensor, y=None, workspace=None, stream=None):
    """y [M, N] bf16 = sa * sb * (a_q [M, K] @ b_q [N, K]^T).

    a_scale: fp32 [M] (per token) or [1]; b_scale: fp32 [N] (per channel) or [1].
    """
    for t, n in ((a_q, "a_q"), (b_q, "b_q")):
        _need(t, torch.float8_e4m3fn, n)
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    _need(a_scale, torch.float32, "a_scale")
    _need(b_scale, torch.float32, "b_scale")
    M, K = a_q.shape
    N = b_q.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=a_q.device)
    if a_scale.numel() not in (1, M) or b_scale.numel() not in (1, N):
        raise ValueError("a_scale must have 1 or M entries, b_scale 1 or N")
    wp, wn, _keep = _ws(workspace, M, N, K, False, a_q.device)
    st = lib.fp8q_scaled_mm(a_q.data_ptr(), b_q.data_ptr(), a_scale.data_ptr(),
                            int(a_scale.numel() == M), b_scale.data_ptr(),
                            int(b_scale.numel() == N), M, N, K, y.data_ptr(), _rowmajor(y, "y"),
                            wp, wn, _stream(stream))
    _check("fp8q_scaled_mm", st)
    return y


def fp8q_scaled_mm_blockwise(a_q: torch.Tensor, b_q: torch.Tensor, a_scale: torch.Tensor,
                             b_scale: torch.Tensor, a_scale_layout: str = "row_major", y=None,
                             workspace=None, stream=None):
    """Block-scaled GEMM: a_scale one fp32 per 1x128 group of A ([M, K/128] row_major or
    [K/128, M] group_major), b_scale fp32 [N/128, K/128]."""
    for t, n in ((a_q, "a_q"), (b_q, "b_q")):
        _need(t, torch.float8_e4m3fn, n)
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    _need(a_scale, torch.float32, "a_scale")
    _need(b_scale, torch.float32, "b_scale")
    M, K = a_q.shape
    N = b_q.shape[0]
    if a_scale_layout == "group_major":
        sm, skb = 1, M
    else:
        sm, skb = K // 128, 1
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=a_q.device)
    wp, wn, _keep = _ws(workspace, M, N, K, True, a_q.device)
    st = lib.fp8q_scaled_mm_blockwise(a_q.data_ptr(), b_q.data_ptr(), a_scale.data_ptr(), sm, skb,
                                      b_scale.data_ptr(), M, N, K, y.data_ptr(),
                                      _rowmajor(y, "y"), wp, wn, _stream(stream))
    _check("fp8q_scaled_mm_blockwise", st)
    return y


def fp8q_scaled_mm_blockwise_e8m0(a_q: torch.Tensor, b_q: torch.Tensor, a_sf: torch.Tensor,
                                  b_sf: torch.Tensor, a_scale_layout: str = "row_major", y=None,
                                  workspace=None, stream=None):
    """Block-scaled GEMM with E8M0 scale bytes (uint8): a_sf one byte per 1x128 group of
    A ([M, K/128] row_major or [K/128, M] group_major), b_sf [N/128, K/128]; the
    tensor core applies the scales (2^(byte - 127))."""
    for t, n in ((a_q, "a_q"), (b_q, "b_q")):
        _need(t, torch.float8_e4m3fn, n)
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    _need(a_sf, torch.uint8, "a_sf")
    _need(b_sf, torch.uint8, "b_sf")
    M, K = a_q.shape
    N = b_q.shape[0]
    sm, skb = (1, M) if a_scale_layout == "group_major" else (K // 128, 1)
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=a_q.device)
    wp, wn, _keep = _ws(workspace, M, N, K, 2, a_q.device)
    st = lib.fp8q_scaled_mm_blockwise_e8m0(a_q.data_ptr(), b_q.data_ptr(), a_sf.data_ptr(), sm,
                                           skb, b_sf.data_ptr(), M, N, K, y.data_ptr(),
                                           _rowmajor(y, "y"), wp, wn, _stream(stream))
    _check("fp8q_scaled_mm_blockwise_e8m0", st)
    return y


def interleave_gate_up(t: torch.Tensor, block: int = 128) -> torch.Tensor:
    """Rows of a gate_up tensor [2I, ...] = [gate (I rows) | up (I rows)] reordered
    into 128-row blocks [gate block 0 | up block 0 | gate block 1 | ...], the
    weight layout fp8q_scaled_mm_blockwise_silu_quant reads (a setup-time
    permutation of the weights; use block=1 for their [2I/128, K/128] scales)."""
    n2 = t.shape[0]
    if n2 % (2 * block):
        raise ValueError(f"rows ({n2}) must be a multiple of {2 * block}")
    nb = n2 // (2 * block)
    rest = t.shape[1:]
    g = t[: n2 // 2].reshape(nb, block, *rest)
    u = t[n2 // 2:].reshape(nb, block, *rest)
    return torch.stack([g, u], dim=1).reshape(n2, *rest).contiguous()


def fp8q_scaled_mm_blockwise_silu_quant(a_q: torch.Tensor, b_q: torch.Tensor, a_scale: torch.Tensor,
                                        b_scale: torch.Tensor, a_scale_layout: str = "row_major",
                                        ue8m0=False, q=None, scales=None,
                                        scale_layout: str = "row_major", stream=None):
    """gate_up blockwise GEMM with the SiLU*mul 1x128 quant fused into its epilogue.
    b_q [2I, K] and b_scale [2I/128, K/128] in the interleaved layout of
    interleave_gate_up.  Returns (q e4m3 [M, I], scales [M, I/128] or [I/128, M]).
    Exact mode: bit-identical to fp8q_scaled_mm_blockwise followed by
    fp8q_silu_mul_quant(h, 128); fast mode (default): the same scales, codes
    within the fused-quant tolerance (fp8q_set_fused_quant_exact)."""
    for t, n in ((a_q, "a_q"), (b_q, "b_q")):
        _need(t, torch.float8_e4m3fn, n)
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    _need(a_scale, torch.float32, "a_scale")
    _need(b_scale, torch.float32, "b_scale")
    M, K = a_q.shape
    N2 = b_q.shape[0]
    I = N2 // 2
    sm, skb = (1, M) if a_scale_layout == "group_major" else (K // 128, 1)
    mode = _ue8m0_mode(ue8m0)
    if q is None:
        q = torch.empty((M, I), dtype=torch.float8_e4m3fn, device=a_q.device)
    scales, ssm, ssg = _scales_out(M, I, 128, scale_layout, a_q.device, scales, mode)
    _check("fp8q_scaled_mm_blockwise_silu_quant", lib.fp8q_scaled_mm_blockwise_silu_quant(
        a_q.data_ptr(), b_q.data_ptr(), a_scale.data_ptr(), sm, skb, b_scale.data_ptr(), M, N2, K, mode,
        q.data_ptr(), _rowmajor(q, "q"), scales.data_ptr(), ssm, ssg, _stream(stream)))
    return q, scales


NOALLOC_SCRATCH_BYTES = 16 << 20


def fp8q_scaled_mm_blockwise_noalloc(a_q: torch.Tensor, b_q: torch.Tensor, a_scale: torch.Tensor,
                                     b_scale: torch.Tensor, a_scale_layout: str = "row_major",
                                     y=None, stream=None):
    """fp8q_scaled_mm_blockwise without a workspace: the library's fixed 16 MiB
    scratch array is used instead (calls that overlap on the GPU race)."""
    for t, n in ((a_q, "a_q"), (b_q, "b_q")):
        _need(t, torch.float8_e4m3fn, n)
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    _need(a_scale, torch.float32, "a_scale")
    _need(b_scale, torch.float32, "b_scale")
    M, K = a_q.shape
    N = b_q.shape[0]
    sm, skb = (1, M) if a_scale_layout == "group_major" else (K // 128, 1)
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=a_q.device)
    st = lib.fp8q_scaled_mm_blockwise_noalloc(a_q.data_ptr(), b_q.data_ptr(), a_scale.data_ptr(),
                                              sm, skb, b_scale.data_ptr(), M, N, K, y.data_ptr(),
                                              _rowmajor(y, "y"), _stream(stream))
    _check("fp8q_scaled_mm_blockwise_noalloc", st)
    return y


# --------------------------------------------------------------- fused_qk_norm_rope
def fp8q_qk_norm_rope(qkv: torch.Tensor, num_heads_q: int, num_heads_k: int, num_heads_v: int,
                      head_dim: int, eps: float, q_weight: torch.Tensor, k_weight: torch.Tensor,
                      cos_sin_cache: torch.Tensor, positions: torch.Tensor, is_neox: bool,
                      stream=None) -> torch.Tensor:
    """In place on qkv (bf16 [T, (hq+hk+hv)*D]): per-head RMSNorm of the q and k heads,
    then the rotary embedding at positions (int64 [T]) from cos_sin_cache (fp32
    [max_pos, D] = cos | sin).  Returns qkv."""
    _need(qkv, torch.bfloat16, "qkv")
    _need(q_weight, torch.bfloat16, "q_weight")
    _need(k_weight, torch.bfloat16, "k_weight")
    _need(cos_sin_cache, torch.float32, "cos_sin_cache")
    _need(positions, torch.int64, "positions")
    if not cos_sin_cache.is_contiguous() or not positions.is_contiguous():
        raise ValueError("cos_sin_cache and positions must be contiguous")
    ld = _rowmajor(qkv, "qkv")
    T = qkv.shape[0]
    _check("fp8q_qk_norm_rope", lib.fp8q_qk_norm_rope(
        qkv.data_ptr(), T, ld, num_heads_q, num_heads_k, num_heads_v, head_dim, ctypes.c_float(eps),
        q_weight.data_ptr(), k_weight.data_ptr(), cos_sin_cache.data_ptr(), cos_sin_cache.shape[0],
        positions.data_ptr(), int(bool(is_neox)), _stream(stream)))
    return qkv


# --------------------------------------------------------------- W8A8_INT8
def _quant_i8_out(M, L, group_size, layout, device, q, scales):
    if q is None:
        q = torch.empty((M, L), dtype=torch.int8, device=device)
    elif q.dtype != torch.int8:
        raise TypeError("q must be int8")
    scales, ssm, ssg = _scales_out(M, L, group_size, layout, device, scales)
    return q, scales, ssm, ssg


def fp8q_group_quant_i8(x: torch.Tensor, group_size: int, q=None, scales=None,
                        scale_layout: str = "row_major", stream=None):
    """W8A8_INT8 quant (group_size = K per token, or 128): int8 codes, scale amax/127."""
    _need(x, torch.bfloat16, "x")
    ldx = _rowmajor(x, "x")
    M, K = x.shape
    q, scales, ssm, ssg = _quant_i8_out(M, K, group_size, scale_layout, x.device, q, scales)
    _check("fp8q_group_quant_i8", lib.fp8q_group_quant_i8(
        x.data_ptr(), M, K, ldx, group_size, q.data_ptr(), _rowmajor(q, "q"), scales.data_ptr(), ssm,
        ssg, _stream(stream)))
    return q, scales


def fp8q_rmsnorm_quant_i8(x: torch.Tensor, w: torch.Tensor, eps: float, group_size: int, q=None,
                          scales=None, scale_layout: str = "row_major", stream=None):
    """RMSNorm + W8A8_INT8 quant."""
    _need(x, torch.bfloat16, "x")
    _need(w, torch.bfloat16, "w")
    ldx = _rowmajor(x, "x")
    M, H = x.shape
    q, scales, ssm, ssg = _quant_i8_out(M, H, group_size, scale_layout, x.device, q, scales)
    _check("fp8q_rmsnorm_quant_i8", lib.fp8q_rmsnorm_quant_i8(
        x.data_ptr(), w.data_ptr(), ctypes.c_float(eps), M, H, ldx, group_size, q.data_ptr(),
        _rowmajor(q, "q"), scales.data_ptr(), ssm, ssg, _stream(stream)))
    return q, scales


def fp8q_silu_mul_quant_i8(x: torch.Tensor, group_size: int, q=None, scales=None,
                           scale_layout: str = "row_major", stream=None):
    """SiLU*mul + W8A8_INT8 quant; x [M, 2I] = [gate | up]."""
    _need(x, torch.bfloat16, "x")
    ldx = _rowmajor(x, "x")
    M, I2 = x.shape
    I = I2 // 2
    q, scales, ssm, ssg = _quant_i8_out(M, I, group_size, scale_layout, x.device, q, scales)
    _check("fp8q_silu_mul_quant_i8", lib.fp8q_silu_mul_quant_i8(
        x.data_ptr(), M, I, ldx, group_size, q.data_ptr(), _rowmajor(q, "q"), scales.data_ptr(), ssm,
        ssg, _stream(stream)))
    return q, scales


def fp8q_scaled_mm_i8(a_q: torch.Tensor, b_q: torch.Tensor, a_scale: torch.Tensor,
                      b_scale: torch.Tensor, y=None, workspace=None, stream=None):
    """W8A8_INT8 GEMM: y [M, N] bf16 = sa * sb * (a_q [M, K] @ b_q [N, K]^T), int8 operands,
    exact integer sums; a_scale fp32 [M] or [1], b_scale fp32 [N] or [1]."""
    for t, n in ((a_q, "a_q"), (b_q, "b_q")):
        _need(t, torch.int8, n)
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    _need(a_scale, torch.float32, "a_scale")
    _need(b_scale, torch.float32, "b_scale")
    M, K = a_q.shape
    N = b_q.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=a_q.device)
    if a_scale.numel() not in (1, M) or b_scale.numel() not in (1, N):
        raise ValueError("a_scale must have 1 or M entries, b_scale 1 or N")
    wp, wn, _keep = _ws(workspace, M, N, K, 3, a_q.device)
    _check("fp8q_scaled_mm_i8", lib.fp8q_scaled_mm_i8(
        a_q.data_ptr(), b_q.data_ptr(), a_scale.data_ptr(), int(a_scale.numel() == M),
        b_scale.data_ptr(), int(b_scale.numel() == N), M, N, K, y.data_ptr(), _rowmajor(y, "y"), wp,
        wn, _stream(stream)))
    return y


def fp8q_select_gemm_variant(M: int, N: int, K: int, blockwise: bool) -> dict:
    v = GemmVariant()
    _check("fp8q_select_gemm_variant", lib.fp8q_select_gemm_variant(M, N, K, int(blockwise),
                                                                    ctypes.byref(v)))
    return v.as_dict()


def fp8q_force_gemm_variant(swap_ab: int | None = None, split_k: int = 1, block_n: int = 128,
                            cta_pair: int = 0):
    """Force a GEMM variant for the following calls (testing/tuning); no args = automatic."""
    if swap_ab is None:
        _check("fp8q_force_gemm_variant", lib.fp8q_force_gemm_variant(None))
        return
    v = GemmVariant(int(swap_ab), int(split_k), int(block_n), int(cta_pair))
    _check("fp8q_force_gemm_variant", lib.fp8q_force_gemm_variant(ctypes.byref(v)))


def fp8q_set_fused_quant_exact(exact: bool) -> None:
    """Arithmetic of the producer-fused quant ops for the calls that follow
    (process-wide): False (default) = fast y within the fused tolerance with
    exact scales, True = bit-exact codes and scales."""
    _check("fp8q_set_fused_quant_exact", lib.fp8q_set_fused_quant_exact(1 if exact else 0))


def fp8q_get_fused_quant_exact() -> bool:
    return bool(lib.fp8q_get_fused_quant_exact())


def fp8q_last_device_status(stream=None) -> int:
    return int(lib.fp8q_last_device_status(_stream(stream)))


def fp8q_status_string(status: int) -> str:
    return lib.fp8q_status_string(status).decode()


def fp8q_version() -> str:
    return lib.fp8q_version().decode()
