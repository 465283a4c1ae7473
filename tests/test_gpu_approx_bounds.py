"""The error bounds the quant kernels' fast paths rest on, measured on this GPU.

The SiLU fast path uses ex2.approx / rcp.approx and the RMSNorm fast path
rsqrtf; their rounding brackets (+-2^-19, +-2^-20) are sized from these
worst-case relative errors: if a bound grew, a fast result could round
differently from the exact value unnoticed.
tests/cuda/approx_bounds.cu checks every fp32 input of the ranges used
against fp64 and reports the maxima.
"""
import os
import shutil
import subprocess

import pytest

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))


def test_hardware_approximation_bounds(tmp_path):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    exe = str(tmp_path / "approx_bounds")
    subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-o", exe,
                    os.path.join(HERE, "cuda", "approx_bounds.cu")], check=True)
    out = subprocess.run([exe], check=True, capture_output=True, text=True, timeout=300).stdout
    ex2, rcp, expf, rsq = (float(v) for v in out.split())
    print(f"ex2.approx {ex2:.3e}, rcp.approx {rcp:.3e}, exp_fast {expf:.3e}, rsqrtf {rsq:.3e}")
    assert ex2 <= 2.0 ** -22.5
    assert rcp <= 2.0 ** -23.0
    assert expf <= 2.0 ** -22.0
    # the SiLU fast value's total relative error must stay inside its bracket
    total = expf + 2.0 ** -24 + rcp + 2 * 2.0 ** -24
    assert total + 2.0 ** -24 < 2.0 ** -19
    # the RMSNorm fast value: rsqrtf + half an ulp (fp32 argument) + one product,
    # inside its +-2^-20 bracket
    assert rsq + 2.0 ** -25 + 2.0 ** -24 + 2.0 ** -24 < 2.0 ** -20
