"""The device-side timeout path of the GEMM, on a GPU, without a fault.

A test-only copy of the library is built with two defines that the shipped
library never has: the TMA producer of the GEMM issues nothing
(FP8Q_TEST_STALL_PRODUCER) and every pipeline wait gives up after 10 ms
(FP8Q_TEST_WAIT_LIMIT_NS).  A GEMM through that copy must come back: the MMA
thread's first wait runs out, the kernel records FP8Q_ERR_TIMEOUT, its other
roles leave on the abort flag, TMEM is released and the kernel returns.  The
status read through the same copy reports the timeout (and clears it), and the
context stays usable: the shipped library then computes a correct GEMM on the
same device.
"""
import ctypes
import importlib.util
import os
import time

import numpy as np
import pytest
import torch

import fp8q_inputs as inp
import oracle
from helpers import bf16_to_np, gemm_tolerance_check, to_dev_codes

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def stalled_lib():
    spec = importlib.util.spec_from_file_location(
        "_fp8q_build", os.path.join(ROOT, "fp8_quantized_linear_rms_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    path = mod.build_variant(os.path.join(ROOT, "_build", "test_timeout"),
                             ["FP8Q_TEST_STALL_PRODUCER=1", "FP8Q_TEST_WAIT_LIMIT_NS=10000000ull"])
    lib = ctypes.CDLL(path)
    P, I64 = ctypes.c_void_p, ctypes.c_int64
    lib.fp8q_scaled_mm.restype = ctypes.c_int
    lib.fp8q_scaled_mm.argtypes = [P, P, P, ctypes.c_int, P, ctypes.c_int, I64, I64, I64, P, I64, P,
                                   ctypes.c_size_t, P]
    lib.fp8q_last_device_status.restype = ctypes.c_int
    lib.fp8q_last_device_status.argtypes = [P]
    return lib


def test_stalled_gemm_times_out_and_the_context_survives(stalled_lib):
    import fp8_quantized_linear_rms_b200 as fq
    M, N, K = 16, 256, 512
    a = inp.random_e4m3_codes(1, (M, K))
    b = inp.random_e4m3_codes(2, (N, K))
    sa, sb = inp.random_scales(3, (M,)), inp.random_scales(4, (N,))
    ad, bd = to_dev_codes(a), to_dev_codes(b)
    sad, sbd = torch.from_numpy(sa).cuda(), torch.from_numpy(sb).cuda()
    y = torch.zeros((M, N), dtype=torch.bfloat16, device="cuda")
    ws = fq.make_workspace(M, N, K, False)
    wsp, wsn = (ws.data_ptr(), ws.numel()) if ws is not None else (None, 0)
    stream = torch.cuda.current_stream().cuda_stream
    assert stalled_lib.fp8q_last_device_status(stream) == fq.OK
    t0 = time.perf_counter()
    st = stalled_lib.fp8q_scaled_mm(ad.data_ptr(), bd.data_ptr(), sad.data_ptr(), 1, sbd.data_ptr(), 1,
                                    M, N, K, y.data_ptr(), N, wsp, wsn, stream)
    assert st == fq.OK                                   # the launch itself succeeds
    assert stalled_lib.fp8q_last_device_status(stream) == fq.ERR_TIMEOUT
    assert time.perf_counter() - t0 < 10.0               # came back after its short limit
    assert stalled_lib.fp8q_last_device_status(stream) == fq.OK     # read clears it
    # the context is still usable: the shipped library computes a correct GEMM
    y2 = fq.fp8q_scaled_mm(ad, bd, sad, sbd, workspace=fq.make_workspace(M, N, K, False))
    torch.cuda.synchronize()
    assert fq.fp8q_last_device_status() == fq.OK
    y_ref, absdot = oracle.scaled_mm(a, b, sa, sb)
    gemm_tolerance_check(bf16_to_np(y2), y_ref, absdot, "after a timeout")
