"""The arithmetic facts the quant kernels' fast paths rest on, measured on this GPU.

The SiLU fast path uses ex2.approx / rcp.approx, its rounding bracket
(+-2^-19) sized from their worst-case relative errors; the RMSNorm path
refines rsqrtf by one Newton step, whose error (1.5 e^2) must stay far below
the 2^-30 margin of its bracket.  tests/cuda/approx_bounds.cu checks every
fp32 input of the ranges used against fp64 and reports the maxima.
The codes come from the IEEE quotient y / s obtained by Markstein's division
step; tests/cuda/quotient_exact.cu checks that against IEEE division for
every bf16 amax and every bf16 y the kernels can meet.
"""
import os
import shutil
import subprocess

import numpy as np
import pytest

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))


def test_hardware_approximation_bounds(tmp_path):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    exe = str(tmp_path / "approx_bounds")
    subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-o", exe,
                    os.path.join(HERE, "cuda", "approx_bounds.cu")], check=True)
    out = subprocess.run([exe], check=True, capture_output=True, text=True, timeout=300).stdout
    ex2, rcp, expf, rsq, rcp_n = (float(v) for v in out.split())
    print(f"ex2.approx {ex2:.3e}, rcp.approx {rcp:.3e}, exp_fast {expf:.3e}, rsqrtf {rsq:.3e}, "
          f"Newton reciprocal {rcp_n:.3e}")
    assert ex2 <= 2.0 ** -22.5
    assert rcp <= 2.0 ** -23.0
    assert expf <= 2.0 ** -22.0
    assert rcp_n <= 2.0 ** -23.9
    # the SiLU fast value p: exp, the rounding of 1 + e, the reciprocal and two
    # products; its bracket ends p (1 -+ 2^-20.5), each rounded once more to
    # fp32, must still enclose the real value
    total = expf + 2.0 ** -24 + rcp_n + 2 * 2.0 ** -24
    lo = float(np.float32(1.0 - 2.0 ** -20.5))
    hi = float(np.float32(1.0 + 2.0 ** -20.5))
    assert lo * (1 + total) * (1 + 2.0 ** -24) < 1.0
    assert hi * (1 - total) * (1 - 2.0 ** -24) > 1.0
    # the RMSNorm r: rsqrtf of the fp32-rounded argument (half an ulp more),
    # one Newton step in fp64 squares the error: far inside the 2^-30 margin
    e = rsq + 2.0 ** -25
    assert 1.5 * e * e + 2.0 ** -50 < 2.0 ** -30


def test_markstein_quotient_equals_ieee_division(tmp_path):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    exe = str(tmp_path / "quotient_exact")
    subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-o", exe,
                    os.path.join(HERE, "cuda", "quotient_exact.cu")], check=True)
    out = subprocess.run([exe], check=True, capture_output=True, text=True, timeout=300).stdout
    bad_q, bad_c = (int(v) for v in out.split())
    assert (bad_q, bad_c) == (0, 0)
