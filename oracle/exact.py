"""Exact-rational brute-force scaled GEMMs -- TEST INFRASTRUCTURE ONLY.

Used to pin the fp64 C oracle on tiny shapes: every e4m3 code and every fp32
scale is a dyadic rational, so sum_k (qa*sa)(qb*sb) has an exact value as a
``fractions.Fraction``.  Codes are decoded with ``ml_dtypes.float8_e4m3fn``
(an independent library), not with the oracle's own decoder.
"""
from __future__ import annotations

from fractions import Fraction

import ml_dtypes
import numpy as np


def decode_e4m3_exact(codes: np.ndarray) -> list:
    vals = np.asarray(codes, np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    return [Fraction(float(v)) for v in vals.reshape(-1)]


def _frac(x) -> Fraction:
    return Fraction(float(np.float32(x)))


def scaled_mm_exact(a_q, b_q, sa, sb):
    """Exact y[m][n] = sum_k (qa[m,k] sa[m])(qb[n,k] sb[n]) as Fractions.

    sa has M entries or 1 (per tensor); sb has N entries or 1.
    """
    a_q = np.asarray(a_q, np.uint8)
    b_q = np.asarray(b_q, np.uint8)
    M, K = a_q.shape
    N, _ = b_q.shape
    A = decode_e4m3_exact(a_q)
    B = decode_e4m3_exact(b_q)
    sa = np.asarray(sa, np.float32).reshape(-1)
    sb = np.asarray(sb, np.float32).reshape(-1)
    out = []
    for m in range(M):
        s_a = _frac(sa[m] if sa.size == M else sa[0])
        row = []
        for n in range(N):
            s_b = _frac(sb[n] if sb.size == N else sb[0])
            acc = Fraction(0)
            for k in range(K):
                acc += (A[m * K + k] * s_a) * (B[n * K + k] * s_b)
            row.append(acc)
        out.append(row)
    return out


def scaled_mm_blockwise_exact(a_q, b_q, sa, sb):
    """Exact y[m][n] = sum_kb sa[m,kb] sb[n//128,kb] sum_{k in block kb} qa qb."""
    a_q = np.asarray(a_q, np.uint8)
    b_q = np.asarray(b_q, np.uint8)
    M, K = a_q.shape
    N, _ = b_q.shape
    KB = K // 128
    A = decode_e4m3_exact(a_q)
    B = decode_e4m3_exact(b_q)
    out = []
    for m in range(M):
        row = []
        for n in range(N):
            acc = Fraction(0)
            for kb in range(KB):
                part = Fraction(0)
                for k in range(kb * 128, (kb + 1) * 128):
                    part += A[m * K + k] * B[n * K + k]
                acc += _frac(sa[m, kb]) * _frac(sb[n // 128, kb]) * part
            row.append(acc)
        out.append(row)
    return out
