"""CUDA-graph capture of the path's calls.

Every entry point is asynchronous on its stream, allocates nothing and never
synchronizes with the host, so a whole decode-sized chain can be captured once
and replayed on new inputs.  Outside a graph each small call pays its launch
and dispatch cost on the CPU, which is why the pages run these kernels under
CUDA graphs ("Helion in vLLM", §"Practical limits"; "Helion linear backend",
§"Cost").  Here the two chains of a Qwen3-style MLP block,

    per token:  RMSNorm-quant -> scaled_mm -> SiLU*mul-quant -> scaled_mm
    blockwise:  RMSNorm-quant -> scaled_mm_blockwise -> SiLU*mul-quant -> scaled_mm_blockwise

are captured into one graph; replays on fresh inputs must reproduce eager
calls on the same inputs bit for bit, for the automatic variants and for
forced split-K and stream-K variants, whose arrival counters must come back
to zero between replays.  (The eager results themselves are checked against
the oracle by the other GPU tests.)

Every kernel is launched with programmatic dependent launch, so it may start
before the previous kernel of the stream has finished and must wait before
reading that kernel's output.  The same chains issued back to back must
therefore equal the chains with a host synchronization after every call,
where no two kernels can overlap.
"""
import numpy as np
import pytest
import torch

import fp8q_inputs as inp
from helpers import to_dev_bf16, to_dev_codes

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import fp8_quantized_linear_rms_b200 as fq   # fails loudly if libfp8q.so is missing

M, H, I = 16, 1024, 512
EPS = 1e-6


class Block:
    """Static buffers of both chains and the calls that fill them."""

    def __init__(self, noalloc: bool):
        dev = torch.device("cuda")
        self.noalloc = noalloc
        self.x = torch.empty((M, H), dtype=torch.bfloat16, device=dev)
        self.w = to_dev_bf16(inp.rms_weight_bf16(701, H))
        self.gu = to_dev_codes(inp.random_e4m3_codes(702, (2 * I, H)))
        self.dn = to_dev_codes(inp.random_e4m3_codes(703, (H, I)))
        self.sgu_bl = torch.from_numpy(inp.random_scales(704, (2 * I // 128, H // 128))).to(dev)
        self.sdn_bl = torch.from_numpy(inp.random_scales(705, (H // 128, I // 128))).to(dev)
        self.sgu_ch = torch.from_numpy(inp.random_scales(706, (2 * I,))).to(dev)
        self.sdn_ch = torch.from_numpy(inp.random_scales(707, (H,))).to(dev)
        e = lambda *s, dt: torch.empty(s, dtype=dt, device=dev)
        f8, bf, f32 = torch.float8_e4m3fn, torch.bfloat16, torch.float32
        self.out = {
            "qa": e(M, H, dt=f8), "sa": e(M, 1, dt=f32), "h": e(M, 2 * I, dt=bf),
            "qh": e(M, I, dt=f8), "sh": e(M, 1, dt=f32), "y": e(M, H, dt=bf),
            "qa_b": e(M, H, dt=f8), "sa_b": e(H // 128, M, dt=f32), "h_b": e(M, 2 * I, dt=bf),
            "qh_b": e(M, I, dt=f8), "sh_b": e(I // 128, M, dt=f32), "y_b": e(M, H, dt=bf),
        }
        if noalloc:
            self.out["y_n"] = e(M, 2 * I, dt=bf)
        self.ws = {
            "gu": fq.make_workspace(M, 2 * I, H, False), "dn": fq.make_workspace(M, H, I, False),
            "gu_b": fq.make_workspace(M, 2 * I, H, True), "dn_b": fq.make_workspace(M, H, I, True),
        }

    def run(self, sync_each=False):
        o, ws = self.out, self.ws
        calls = [
            lambda: fq.fp8q_rmsnorm_quant(self.x, self.w, EPS, H, q=o["qa"], scales=o["sa"]),
            lambda: fq.fp8q_scaled_mm(o["qa"], self.gu, o["sa"].view(-1), self.sgu_ch, y=o["h"],
                                      workspace=ws["gu"]),
            lambda: fq.fp8q_silu_mul_quant(o["h"], I, q=o["qh"], scales=o["sh"]),
            lambda: fq.fp8q_scaled_mm(o["qh"], self.dn, o["sh"].view(-1), self.sdn_ch, y=o["y"],
                                      workspace=ws["dn"]),
            lambda: fq.fp8q_rmsnorm_quant(self.x, self.w, EPS, 128, q=o["qa_b"], scales=o["sa_b"],
                                          scale_layout="group_major"),
            lambda: fq.fp8q_scaled_mm_blockwise(o["qa_b"], self.gu, o["sa_b"], self.sgu_bl,
                                                a_scale_layout="group_major", y=o["h_b"],
                                                workspace=ws["gu_b"]),
            lambda: fq.fp8q_silu_mul_quant(o["h_b"], 128, q=o["qh_b"], scales=o["sh_b"],
                                           scale_layout="group_major"),
            lambda: fq.fp8q_scaled_mm_blockwise(o["qh_b"], self.dn, o["sh_b"], self.sdn_bl,
                                                a_scale_layout="group_major", y=o["y_b"],
                                                workspace=ws["dn_b"]),
        ]
        if self.noalloc:
            calls.append(lambda: fq.fp8q_scaled_mm_blockwise_noalloc(
                o["qa_b"], self.gu, o["sa_b"], self.sgu_bl, a_scale_layout="group_major",
                y=o["y_n"]))
        for c in calls:
            c()
            if sync_each:
                torch.cuda.synchronize()

    def snapshot(self) -> dict:
        torch.cuda.synchronize()
        return {k: v.view(torch.uint8).cpu().numpy().copy() if v.dtype == torch.float8_e4m3fn
                else v.cpu().numpy().copy() if v.dtype == torch.float32
                else v.view(torch.int16).cpu().numpy().copy()
                for k, v in self.out.items()}


def _inputs(seed):
    return to_dev_bf16(inp.heavy_tailed_bf16(seed, M, H))


def _assert_same(a: dict, b: dict, what: str):
    for k in a:
        assert np.array_equal(a[k], b[k]), f"{what}: {k} differs"


@pytest.mark.parametrize("variant", [None, (1, 4, 16), (1, 0, 16), (0, 2, 128)],
                         ids=["auto", "swap-splitk4", "swap-streamk", "splitk2"])
def test_chain_replays_in_a_cuda_graph(variant):
    if variant is None:
        fq.fp8q_force_gemm_variant()
    else:
        fq.fp8q_force_gemm_variant(*variant)
    try:
        blk = Block(noalloc=variant is None)   # the no-allocation entry takes no forced variant
        x1, x2 = _inputs(711), _inputs(712)
        # eager references
        blk.x.copy_(x1)
        blk.run()
        e1 = blk.snapshot()
        blk.x.copy_(x2)
        blk.run()
        e2 = blk.snapshot()
        # capture (warm-up on a side stream first, as torch requires)
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            blk.run()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            blk.run()
        for x, ref, what in ((x1, e1, "replay on x1"), (x2, e2, "replay on x2"),
                             (x1, e1, "second replay on x1")):
            for t in blk.out.values():
                t.view(torch.uint8).fill_(0xFF)        # stale outputs would show
            blk.x.copy_(x)
            g.replay()
            _assert_same(ref, blk.snapshot(), what)
        assert fq.fp8q_last_device_status() == fq.OK
        del g
    finally:
        fq.fp8q_force_gemm_variant()


@pytest.mark.parametrize("variant", [None, (1, 4, 16), (0, 2, 128)],
                         ids=["auto", "swap-splitk4", "splitk2"])
def test_back_to_back_calls_match_serialized_calls(variant):
    if variant is None:
        fq.fp8q_force_gemm_variant()
    else:
        fq.fp8q_force_gemm_variant(*variant)
    try:
        blk = Block(noalloc=variant is None)
        for seed in (721, 722):
            blk.x.copy_(_inputs(seed))
            torch.cuda.synchronize()
            blk.run(sync_each=True)
            ref = blk.snapshot()
            for rep in range(3):
                # poison every intermediate and output, then the chain with no
                # host sync: a kernel reading its producer's output too early
                # would see the poison
                for t in blk.out.values():
                    t.view(torch.uint8).fill_(0xFF)
                blk.run()
                _assert_same(ref, blk.snapshot(), f"back-to-back chain, input {seed}, run {rep}")
        assert fq.fp8q_last_device_status() == fq.OK
    finally:
        fq.fp8q_force_gemm_variant()
