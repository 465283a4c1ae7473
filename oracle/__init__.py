"""CPU oracle of the FP8 W8A8 linear path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never calls it and
shares no code with it.  The arithmetic lives in ``fp8q_oracle.c`` (plain C,
fp64 unless the definition fixes fp32); this module compiles it with gcc and
marshals numpy arrays through ctypes.  ``exact.py`` holds an exact-rational
brute-force GEMM used to pin the C GEMM on tiny shapes.

All bf16 tensors cross this interface as ``numpy.uint16`` bit patterns; codes
as ``numpy.uint8`` e4m3fn bytes; scales as ``numpy.float32``; GEMM references
as ``numpy.float64``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fp8q_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ``fp8q_oracle.c`` into ``liboracle.so`` (gcc, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
               "-fno-fast-math", _SRC, "-o", _LIB + ".tmp", "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i64 = ctypes.c_int64
        lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        lib.oracle_e4m3_encode.restype = ctypes.c_uint8
        lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_decode.restype = ctypes.c_double
        lib.oracle_bf16_round.argtypes = [ctypes.c_double]
        lib.oracle_bf16_round.restype = ctypes.c_float
        lib.oracle_scale.argtypes = [ctypes.c_float, ctypes.c_int]
        lib.oracle_scale.restype = ctypes.c_float
        lib.oracle_group_quant.argtypes = [P, i64, i64, i64, i64, ctypes.c_int, P, P, P]
        lib.oracle_rmsnorm_quant.argtypes = [P, P, ctypes.c_float, i64, i64, i64, i64,
                                             ctypes.c_int, P, P, P]
        lib.oracle_silu_mul_quant.argtypes = [P, i64, i64, i64, i64, ctypes.c_int, P, P, P]
        lib.oracle_add_rmsnorm_quant.argtypes = [P, P, P, ctypes.c_float, i64, i64, i64,
                                                 ctypes.c_int, P, P, P, P]
        lib.oracle_scaled_mm_rows.argtypes = [P, P, P, ctypes.c_int, P, ctypes.c_int, i64, i64,
                                              i64, P, i64, P, P]
        lib.oracle_scaled_mm_blockwise_rows.argtypes = [P, P, P, P, i64, i64, i64, P, i64, P, P]
        lib.oracle_e4m3_encode_array.argtypes = [P, i64, P]
        lib.oracle_e4m3_decode_array.argtypes = [P, i64, P]
        lib.oracle_bf16_round_array.argtypes = [P, i64, P]
        lib.oracle_scale_array.argtypes = [P, i64, ctypes.c_int, P]
        lib.oracle_int8_quant_rows.argtypes = [P, i64, i64, i64, P, P]
        lib.oracle_scaled_mm_i8_rows.argtypes = [P, P, P, ctypes.c_int, P, ctypes.c_int, i64, i64,
                                                 i64, P, i64, P, P]
        lib.oracle_int8_encode.argtypes = [ctypes.c_float]
        lib.oracle_int8_encode.restype = ctypes.c_int8
        lib.oracle_int8_scale.argtypes = [ctypes.c_float]
        lib.oracle_int8_scale.restype = ctypes.c_float
        lib.oracle_qk_norm_rope.argtypes = [P, i64, i64, i64, i64, i64, ctypes.c_float, P, P, P, P,
                                            ctypes.c_int]
        lib.oracle_e8m0_encode_array.argtypes = [P, i64, P]
        lib.oracle_e8m0_decode_array.argtypes = [P, i64, P]
        for f in ("oracle_group_quant", "oracle_rmsnorm_quant", "oracle_silu_mul_quant",
                  "oracle_add_rmsnorm_quant",
                  "oracle_scaled_mm_rows", "oracle_scaled_mm_blockwise_rows",
                  "oracle_e4m3_encode_array", "oracle_e4m3_decode_array",
                  "oracle_bf16_round_array", "oracle_scale_array", "oracle_e8m0_encode_array",
                  "oracle_e8m0_decode_array", "oracle_int8_quant_rows", "oracle_scaled_mm_i8_rows",
                  "oracle_qk_norm_rope"):
            getattr(lib, f).restype = None
        _lib = lib
    return _lib


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# --------------------------------------------------------------------- formats
def e4m3_encode(v) -> np.ndarray:
    """Saturating round-to-nearest-even e4m3fn codes of fp32 values."""
    v = _c(v, np.float32)
    out = np.empty(v.shape, np.uint8)
    _load().oracle_e4m3_encode_array(_ptr(v), v.size, _ptr(out))
    return out


def e4m3_decode(c) -> np.ndarray:
    c = _c(c, np.uint8)
    out = np.empty(c.shape, np.float64)
    _load().oracle_e4m3_decode_array(_ptr(c), c.size, _ptr(out))
    return out


def bf16_round(v) -> np.ndarray:
    """Nearest-even bfloat16 of fp64 values, returned as float32."""
    v = _c(v, np.float64)
    out = np.empty(v.shape, np.float32)
    _load().oracle_bf16_round_array(_ptr(v), v.size, _ptr(out))
    return out


def scale(amax, ue8m0: bool = False) -> np.ndarray:
    a = _c(amax, np.float32)
    out = np.empty(a.shape, np.float32)
    _load().oracle_scale_array(_ptr(a), a.size, int(ue8m0), _ptr(out))
    return out


def e8m0_encode(s) -> np.ndarray:
    """E8M0 bytes of power-of-two fp32 scales (255 for anything that is not a
    power of two in [2^-127, 2^127])."""
    s = _c(s, np.float32)
    out = np.empty(s.shape, np.uint8)
    _load().oracle_e8m0_encode_array(_ptr(s), s.size, _ptr(out))
    return out


def e8m0_decode(b) -> np.ndarray:
    """Values 2^(b - 127) of E8M0 bytes (NaN for 255), as float64."""
    b = _c(b, np.uint8)
    out = np.empty(b.shape, np.float64)
    _load().oracle_e8m0_decode_array(_ptr(b), b.size, _ptr(out))
    return out


def _packed(res, ue8m0):
    """For ue8m0 == "packed": the UE8M0 scales as E8M0 bytes."""
    if ue8m0 != "packed":
        return res
    return (res[0], e8m0_encode(res[1])) + tuple(res[2:])


# ---------------------------------------------------------------- quant ops
def _quant_out(M, L, g, want_y):
    q = np.empty((M, L), np.uint8)
    s = np.empty((M, L // g), np.float32)
    y = np.empty((M, L), np.float32) if want_y else None
    return q, s, y


def _check_group(L, g):
    if g <= 0 or L % g != 0:
        raise ValueError(f"group size {g} does not divide row length {L}")


def group_quant(x_bits: np.ndarray, group_size: int, ue8m0: bool = False, want_y: bool = False):
    """per_token_group_fp8_quant (group_size=128) / per-token quant (group_size=K).

    x_bits: uint16 bf16 bits [M, K].  Returns (q [M,K] uint8, s [M,K/g] f32[, y]).
    """
    x = _c(x_bits, np.uint16)
    M, K = x.shape
    _check_group(K, group_size)
    q, s, y = _quant_out(M, K, group_size, want_y)
    _load().oracle_group_quant(_ptr(x), M, K, K, group_size, int(bool(ue8m0)), _ptr(q), _ptr(s),
                               _ptr(y))
    return _packed((q, s, y) if want_y else (q, s), ue8m0)


def rmsnorm_quant(x_bits, w_bits, eps: float, group_size: int, ue8m0: bool = False,
                  want_y: bool = False):
    """rms_norm_dynamic_per_token_quant (g=H) / rms_norm_per_block_quant (g=128)."""
    x = _c(x_bits, np.uint16)
    w = _c(w_bits, np.uint16)
    M, H = x.shape
    assert w.shape == (H,)
    _check_group(H, group_size)
    q, s, y = _quant_out(M, H, group_size, want_y)
    _load().oracle_rmsnorm_quant(_ptr(x), _ptr(w), ctypes.c_float(eps), M, H, H, group_size,
                                 int(bool(ue8m0)), _ptr(q), _ptr(s), _ptr(y))
    return _packed((q, s, y) if want_y else (q, s), ue8m0)


def add_rmsnorm_quant(x_bits, res_bits, w_bits, eps: float, group_size: int, ue8m0=False,
                      want_y: bool = False):
    """Residual add + RMSNorm quant: h = bf16(x + residual) (returned as the
    updated residual), then rmsnorm_quant(h).  Returns (q, s, residual_out[, y])."""
    x = _c(x_bits, np.uint16)
    r = _c(res_bits, np.uint16)
    w = _c(w_bits, np.uint16)
    M, H = x.shape
    assert r.shape == (M, H) and w.shape == (H,)
    _check_group(H, group_size)
    q, s, y = _quant_out(M, H, group_size, want_y)
    r_out = np.empty((M, H), np.uint16)
    _load().oracle_add_rmsnorm_quant(_ptr(x), _ptr(r), _ptr(w), ctypes.c_float(eps), M, H,
                                     group_size, int(bool(ue8m0)), _ptr(q), _ptr(s), _ptr(r_out),
                                     _ptr(y))
    res = (q, s, r_out, y) if want_y else (q, s, r_out)
    return _packed(res, ue8m0)


def silu_mul_quant(x_bits, group_size: int, ue8m0: bool = False, want_y: bool = False):
    """silu_and_mul_dynamic_per_token_quant (g=I) / silu_and_mul_per_block_quant (g=128).

    x_bits: [M, 2I] = [gate | up].
    """
    x = _c(x_bits, np.uint16)
    M, I2 = x.shape
    assert I2 % 2 == 0
    I = I2 // 2
    _check_group(I, group_size)
    q, s, y = _quant_out(M, I, group_size, want_y)
    _load().oracle_silu_mul_quant(_ptr(x), M, I, I2, group_size, int(bool(ue8m0)), _ptr(q),
                                  _ptr(s), _ptr(y))
    return _packed((q, s, y) if want_y else (q, s), ue8m0)


# ---------------------------------------------------------------------- GEMMs
def _rows(M, rows):
    if rows is None:
        rows = np.arange(M, dtype=np.int64)
    rows = _c(rows, np.int64)
    assert rows.ndim == 1 and (rows.size == 0 or (rows.min() >= 0 and rows.max() < M))
    return rows


def scaled_mm(a_q, b_q, sa, sb, rows=None):
    """fp64 reference of scaled_mm for the listed rows of A.

    a_q [M,K] uint8, b_q [N,K] uint8, sa: [M] (per token) or [1] (per tensor),
    sb: [N] (per channel) or [1] (per tensor).  Returns (y_ref, absdot), both
    [len(rows), N] float64.
    """
    a = _c(a_q, np.uint8)
    b = _c(b_q, np.uint8)
    M, K = a.shape
    N, K2 = b.shape
    assert K == K2
    sa = _c(sa, np.float32).reshape(-1)
    sb = _c(sb, np.float32).reshape(-1)
    assert sa.size in (1, M) and sb.size in (1, N)
    rows = _rows(M, rows)
    y = np.empty((rows.size, N), np.float64)
    ad = np.empty((rows.size, N), np.float64)
    _load().oracle_scaled_mm_rows(_ptr(a), _ptr(b), _ptr(sa), int(sa.size == M), _ptr(sb), int(sb.size == N), M, N, K,
                                  _ptr(rows), rows.size, _ptr(y), _ptr(ad))
    return y, ad


def scaled_mm_blockwise(a_q, b_q, sa, sb, rows=None):
    """fp64 reference of scaled_mm_blockwise for the listed rows of A.

    sa [M, K/128] (row-major, one scale per 1x128 group of A), sb [N/128, K/128].
    """
    a = _c(a_q, np.uint8)
    b = _c(b_q, np.uint8)
    M, K = a.shape
    N, K2 = b.shape
    assert K == K2 and K % 128 == 0 and N % 128 == 0
    sa = _c(sa, np.float32)
    sb = _c(sb, np.float32)
    assert sa.shape == (M, K // 128) and sb.shape == (N // 128, K // 128)
    rows = _rows(M, rows)
    y = np.empty((rows.size, N), np.float64)
    ad = np.empty((rows.size, N), np.float64)
    _load().oracle_scaled_mm_blockwise_rows(_ptr(a), _ptr(b), _ptr(sa), _ptr(sb), M, N, K,
                                            _ptr(rows), rows.size, _ptr(y), _ptr(ad))
    return y, ad


def scaled_mm_blockwise_e8m0(a_q, b_q, sa_e8m0, sb_e8m0, rows=None):
    """scaled_mm_blockwise with E8M0 scale bytes: sa [M, K/128], sb [N/128, K/128]
    (uint8), each byte b standing for the scale 2^(b - 127)."""
    sa = e8m0_decode(sa_e8m0).astype(np.float32)
    sb = e8m0_decode(sb_e8m0).astype(np.float32)
    return scaled_mm_blockwise(a_q, b_q, sa, sb, rows)


# --------------------------------------------------------------------- W8A8_INT8
def int8_quantize(y, group_size: int):
    """int8 codes and fp32 scales of fp32 values y [M, L] in groups of g:
    s = fl32(max(amax, 1e-10)/127), q = sat_int8(RNE(fl32(y/s)))."""
    y = _c(y, np.float32)
    M, L = y.shape
    _check_group(L, group_size)
    q = np.empty((M, L), np.int8)
    s = np.empty((M, L // group_size), np.float32)
    _load().oracle_int8_quant_rows(_ptr(y), M, L, group_size, _ptr(q), _ptr(s))
    return q, s


def int8_encode_scalar(v: float) -> int:
    return int(_load().oracle_int8_encode(ctypes.c_float(v)))


def group_quant_i8(x_bits, group_size: int):
    """W8A8_INT8 per-token (g = K) / per-group quant of bf16 x: (q int8, s fp32)."""
    _, _, y = group_quant(x_bits, group_size, False, want_y=True)
    return int8_quantize(y, group_size)


def rmsnorm_quant_i8(x_bits, w_bits, eps: float, group_size: int):
    """RMSNorm (same reading as rmsnorm_quant) followed by int8 quant."""
    _, _, y = rmsnorm_quant(x_bits, w_bits, eps, group_size, False, want_y=True)
    return int8_quantize(y, group_size)


def silu_mul_quant_i8(x_bits, group_size: int):
    """SiLU*mul (same reading as silu_mul_quant) followed by int8 quant."""
    _, _, y = silu_mul_quant(x_bits, group_size, False, want_y=True)
    return int8_quantize(y, group_size)


def scaled_mm_i8(a_q, b_q, sa, sb, rows=None):
    """fp64 reference of the int8 scaled_mm for the listed rows of A: the
    integer dot products exact, then times sa (per token or per tensor) and
    sb (per channel or per tensor).  Returns (y_ref, absdot)."""
    a = _c(a_q, np.int8)
    b = _c(b_q, np.int8)
    M, K = a.shape
    N, K2 = b.shape
    assert K == K2
    sa = _c(sa, np.float32).reshape(-1)
    sb = _c(sb, np.float32).reshape(-1)
    assert sa.size in (1, M) and sb.size in (1, N)
    rows = _rows(M, rows)
    y = np.empty((rows.size, N), np.float64)
    ad = np.empty((rows.size, N), np.float64)
    _load().oracle_scaled_mm_i8_rows(_ptr(a), _ptr(b), _ptr(sa), int(sa.size == M), _ptr(sb),
                                     int(sb.size == N), M, N, K, _ptr(rows), rows.size, _ptr(y),
                                     _ptr(ad))
    return y, ad


# --------------------------------------------------------------- fused_qk_norm_rope
def qk_norm_rope(qkv_bits, hq: int, hk: int, hv: int, head_dim: int, eps: float, q_w_bits, k_w_bits,
                 cos_sin, positions, is_neox: bool):
    """Per-head RMSNorm of the q and k heads, then the rotary embedding at each
    token's position; returns a new qkv (uint16 bf16 bits [T, (hq+hk+hv)*D]),
    v heads unchanged.  cos_sin: fp32 [max_pos, D] = [cos (D/2) | sin (D/2)]."""
    x = np.array(qkv_bits, dtype=np.uint16, copy=True, order="C")
    T, L = x.shape
    D = head_dim
    assert L == (hq + hk + hv) * D and D % 2 == 0
    qw = _c(q_w_bits, np.uint16)
    kw = _c(k_w_bits, np.uint16)
    cs = _c(cos_sin, np.float32)
    pos = _c(positions, np.int64)
    assert qw.shape == (D,) and kw.shape == (D,) and cs.shape[1] == D and pos.shape == (T,)
    assert pos.size == 0 or (pos.min() >= 0 and pos.max() < cs.shape[0])
    _load().oracle_qk_norm_rope(_ptr(x), T, L, hq, hk, D, ctypes.c_float(eps), _ptr(qw), _ptr(kw),
                                _ptr(cs), _ptr(pos), int(bool(is_neox)))
    return x


# ----------------------------------------------- gate_up GEMM + SiLU*mul quant (fused)
def gate_up_silu_quant(a_q, b_q, sa, sb, group_size: int = 128, ue8m0=False, rows=None):
    """The fused op's definition, written as the chain it replaces: the blockwise
    gate_up GEMM (rows of A; W = [gate (I rows) | up (I rows)], block scales),
    each output rounded to bf16 as the GEMM emits it, then SiLU*mul quant of
    h = [h_gate | h_up].  Returns (q, s, h_bits) for the listed rows."""
    y, _ = scaled_mm_blockwise(a_q, b_q, sa, sb, rows)
    h = bf16_round(y)
    h_bits = (h.view(np.uint32) >> 16).astype(np.uint16)
    res = silu_mul_quant(h_bits, group_size, ue8m0)
    return res + (h_bits,)
