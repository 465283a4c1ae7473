#!/usr/bin/env python
"""Benchmark of the FP8 W8A8 linear path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--m M] [--impl reference]
                    [--no-e8m0] [--sweep quant|gemm8b|decode32b|prefill32b|library|all|oracle]

Workload: the linear stack of one Qwen3-32B-shaped decoder block in prefill
(hidden 5120, intermediate 25600, 64 query / 8 kv heads of 128) on a batch of
M = 8192 tokens, through both FP8 schemes.  One step runs, per scheme,
    rmsnorm_quant(x)        -> scaled_mm qkv      [5120 -> 10240]
    group_quant(attn)       -> scaled_mm o        [8192 -> 5120]
    rmsnorm_quant(o out)    -> scaled_mm gate_up  [5120 -> 51200]
    silu_mul_quant(gate_up) -> scaled_mm down     [25600 -> 5120]
with per-token activation scales and per-channel weight scales (scaled_mm),
then with 1x128 activation groups and 128x128 weight blocks
(scaled_mm_blockwise, fp32 scales), where the gate_up GEMM and the SiLU*mul
quant run as one fused launch (scaled_mm_blockwise_silu_quant: the 2I-wide
bf16 intermediate is never written): 15 launches.  The attention output that
feeds the o projection is a seeded stand-in (attention itself is not part of
this path).  x is heavy-tailed Student-t(3) with 1% outlier channels x20,
attn ~ N(0, 1) (seeded); weights W ~ N(0, 0.02), quantized once per output
channel / per 128x128 block.

`value` is whole-job TFLOP/s (GEMM FLOPs of all ranks / max-over-ranks device
time), inputs resident in HBM; each timed step is bracketed by CUDA events,
every launch of the step is followed by an event (the per-kernel times), and
an untimed 256 MiB write flushes L2 between steps.  `e2e` is the same metric
through the public API with each step's inputs copied from pinned host memory
and its two block outputs copied back inside the timed region, the copies on
their own streams overlapping the neighbouring steps' kernels
(double-buffered, as a serving loop runs).  `roofline` is the dominant kernel
(the launch with the largest device time), `gemms` and `roofline_quant` every
GEMM and quant launch against the measured peaks.  `e8m0_chain` times the
blockwise stack again with packed UE8M0 scales and the block-scaled GEMM;
`qk_norm_rope` times the attention-side fused op on the step's qkv output.
The quant ops run in the library's default arithmetic: the per-token SiLU*mul
quant and the SiLU*mul quant fused into the gate_up GEMM keep exact scales
with codes within the fused tolerance, the others are bit-exact;
fp8q_set_fused_quant_exact makes all of them bit-exact.
`--impl reference` times the CPU oracle on a bounded sample of the workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

# Qwen3-32B block: hidden, intermediate, attention width (64 heads x 128)
H, I, ATT = 5120, 25600, 8192
QKV = (64 + 2 * 8) * 128
LAYERS = (("qkv", H, QKV), ("o", ATT, H), ("gate_up", H, 2 * I), ("down", I, H))   # (name, K, N)
DEFAULT_M = 8192
METRIC = "FP8 quant+scaled_mm TFLOP/s (Qwen3-32B prefill linear stack, per-token + blockwise)"
EPS = 1e-6
NOMINAL_FP8_TFLOPS = 4500.0      # dense e4m3 tensor peak on the data sheet, for context beside `frac`

# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of
# the step's dominant kernel, from one ncu capture of the full-size launch
# (`ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum -k regex:gemm_
# -s 6 -c 1` on `bench.py --steps 1 --warmup 3 --no-e8m0 --no-rope`, the
# seventh GEMM launch being the fused gate_up).  It holds for the GEMM code
# it was taken on: the line reports it only while the SHA-256 digest of that
# code (comments and blank space dropped) is unchanged, else null.
GEMM_SOURCES = ("fp8q_gemm.cu", "fp8q_sm100.cuh", "fp8q_quant_math.cuh", "fp8q_common.cuh")
TRAFFIC_CAPTURES = {
    ("scaled_mm_blockwise_silu_quant", 8192): {
        "read": 374152960, "write": 211215616,
        "sources_sha256": "8cfca17b2a9d48b32d4f7278dc1d43b35810671a4314e026bcbe53cba4d81ac5"},
}


def gemm_sources_digest():
    """SHA-256 of the GEMM sources' code: comments and blank space dropped, so
    that an edit of a comment keeps a capture valid and any code edit does not."""
    import hashlib
    import re
    h = hashlib.sha256()
    for f in GEMM_SOURCES:
        with open(os.path.join(ROOT, "fp8_quantized_linear_rms_b200", "csrc", f)) as fh:
            src = fh.read()
        src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)    # block comments
        src = re.sub(r"//[^\n]*", " ", src)                  # line comments
        h.update(" ".join(src.split()).encode())
    return h.hexdigest()


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--m", type=int, default=DEFAULT_M)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-e8m0", action="store_true", help="skip the E8M0 (UE8M0) chain")
    ap.add_argument("--no-rope", action="store_true", help="skip timing fused_qk_norm_rope")
    ap.add_argument("--sweep", default=None,
                    help="per-op timing instead of the step: quant, gemm8b, decode32b, prefill32b, library, "
                         "e8m0, all (GPU), or oracle (the CPU oracle, all host cores and one core)")
    ap.add_argument("--reps", type=int, default=50)
    ap.add_argument("--sweep-m", default=None,
                    help="comma-separated token counts replacing each sweep's own list of M")
    return ap.parse_args()


def gemm_flops(M):
    """GEMM FLOPs of one step: both schemes x the four layers."""
    return 2 * sum(2 * M * N * K for _, K, N in LAYERS)


def fused_gate_up_bytes(M):
    """Algorithmic HBM bytes of the fused gate_up + SiLU*mul 1x128 quant launch:
    e4m3 activations and weights and their fp32 block scales read once, e4m3
    codes [M, I] and fp32 group scales written once."""
    K, N2 = H, 2 * I
    return (M * K + N2 * K + 4 * M * (K // 128) + 4 * (N2 // 128) * (K // 128)
            + M * I + 4 * M * (I // 128))


def quant_bytes(op, M, L, g):
    """Algorithmic HBM bytes of one quant launch over M rows of length L (the
    row length of the quantized values) in groups of g: the bf16 input read
    once, e4m3 codes and fp32 scales written once, the RMSNorm weight once."""
    if op == "silu_mul_quant":
        return M * (4 * L + L + 4 * (L // g))
    b = M * (2 * L + L + 4 * (L // g))
    return b + 2 * L if op == "rmsnorm_quant" else b


def max_over_ranks(values, world, device="cpu"):
    """Element-wise maximum of each rank's timings, returned on every rank (the
    slowest rank sets the job's time)."""
    import torch
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_tflops(flops_per_rank_step, steps, world, ms):
    """Whole-job throughput: the GEMM FLOPs all ranks did in `steps` steps over
    the (max-over-ranks) time `ms`; each rank runs its own batch (replicas)."""
    return flops_per_rank_step * steps * world / (ms * 1e-3) / 1e12


def workload_config(M, n):
    return {"workload": f"qwen3-32b-prefill-m{M}-linear-stack-per-token+blockwise",
            "model": "Qwen3-32B-shaped decoder block linears (hidden 5120, intermediate 25600, "
                     "64 q / 8 kv heads of 128): qkv, o, gate_up, down",
            "global_batch": M * n, "tokens_per_gpu": M, "seq_len": None,
            "parallelism": f"replicas{n}" if n > 1 else "single-gpu",
            "l2": "flushed between timed steps (256 MiB write); the step's weights "
                  "(0.98 GB of e4m3) exceed L2 as well",
            "fused_quant": "library default (fast mode): the per-token SiLU*mul quant and the "
                           "SiLU*mul quant fused into the gate_up GEMM keep exact scales, codes "
                           "within the fused tolerance; the other quant ops bit-exact"}


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f)
    except Exception:
        return {}


def fp8_peak(peaks, timed_s):
    """Dense FP8 denominator: 2 x the measured bf16 GEMM rate (nominal fp8:bf16
    = 4.5:2.25); the burst figure for a timed region under a second, the
    sustained one (measured over seconds under the power cap) beyond."""
    burst, sust = peaks.get("bf16_tflops"), peaks.get("bf16_tflops_sustained")
    if timed_s >= 1.0:
        if sust:
            return 2.0 * sust, f"of measured: 2 x bf16 sustained (timed region {timed_s:.2f} s)"
        return 2.0 * 1400.0, "of fallback: 2 x 1.4 PF bf16 sustained"
    if burst:
        return 2.0 * burst, f"of measured: 2 x bf16 burst (timed region {timed_s:.2f} s)"
    return 2.0 * 1590.0, "of fallback: 2 x 1.59 PF bf16 burst"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """SM clock and throttle reasons sampled every 10 ms during the timed
    region (NVML; nvidia-smi at 200 ms when NVML is unavailable)."""

    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4}

    def __init__(self, index):
        self.index = index
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self._proc = None

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))

            def run():
                while not self._stop.is_set():
                    try:
                        self.samples.append(float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)))
                        r = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                        for nm, bit in self.REASONS.items():
                            if r & bit:
                                self.reasons.add(nm)
                    except Exception:
                        pass
                    self._stop.wait(0.01)

            self._thread = threading.Thread(target=run, daemon=True)
            self._thread.start()
        except Exception:
            self._thread = None
            self._start_smi()

    def _start_smi(self):
        import tempfile
        self.path = os.path.join(tempfile.gettempdir(), f"fp8q_clocks_{os.getpid()}.csv")
        try:
            self.f = open(self.path, "w")
            self._proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}",
                 "--query-gpu=clocks.sm,clocks.max.sm,clocks_event_reasons.active,"
                 "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                 "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self._proc = None
            if getattr(self, "f", None):
                self.f.close()
                os.remove(self.path)

    def stop(self):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=5)
        elif self._proc is not None:
            self._proc.terminate()
            try:
                self._proc.wait(timeout=5)
            except Exception:
                self._proc.kill()
            self.f.close()
            names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
            with open(self.path) as f:
                for line in f:
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) < 7:
                        continue
                    try:
                        self.samples.append(float(parts[0]))
                        self.max_mhz = max(self.max_mhz or 0.0, float(parts[1]))
                    except ValueError:
                        continue
                    for nm, v in zip(names, parts[3:7]):
                        if v.lower() == "active":
                            self.reasons.add(nm)
            os.remove(self.path)
        if not self.samples:
            return None
        srt = sorted(self.samples)
        return {"sm_mhz": statistics.median(srt), "sm_max_mhz": self.max_mhz,
                "sm_mhz_min": srt[0], "sm_mhz_p10": srt[len(srt) // 10],
                "reasons": sorted(self.reasons), "samples": len(srt)}


# ------------------------------------------------------------------ native arm
def run_native(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import fp8_quantized_linear_rms_b200 as fq
    import fp8q_inputs as inp

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    M = args.m
    torch.manual_seed(1234 + rank)

    def host_bf16(bits):
        return torch.from_numpy(bits.view("int16")).view(torch.bfloat16)

    # ---- inputs (seeded, synthetic) and weights, resident in HBM
    x_host = host_bf16(inp.heavy_tailed_bf16(2000 + rank, M, H))
    a_host = host_bf16(inp.normal_bf16(2100 + rank, (M, ATT)))
    x_pinned, a_pinned = x_host.pin_memory(), a_host.pin_memory()
    x, attn = x_host.to(dev), a_host.to(dev)
    w_in = host_bf16(inp.rms_weight_bf16(2001, H)).to(dev)
    w_post = host_bf16(inp.rms_weight_bf16(2002, H)).to(dev)

    def make_weight(N, K, seed):
        g = torch.Generator(device=dev).manual_seed(seed)
        return (torch.randn(N, K, generator=g, device=dev) * 0.02).to(torch.bfloat16)

    def per_channel(W):
        q, s = fq.fp8q_group_quant(W, W.shape[1])
        return q, s.reshape(-1).contiguous()

    def per_block(W, pow2=False):
        # weight block scales: amax of each 128x128 block / 448 (setup, untimed)
        N, K = W.shape
        wb = W.float().view(N // 128, 128, K // 128, 128)
        s = (wb.abs().amax(dim=(1, 3)).clamp_min(1e-10) / 448.0).float()
        if pow2:
            s = torch.pow(2.0, torch.ceil(torch.log2(s)))
        q = (wb / s[:, None, :, None]).clamp(-448, 448).to(torch.float8_e4m3fn).view(N, K)
        return q.contiguous(), s.contiguous()

    f8 = torch.float8_e4m3fn
    W = {}
    for i, (name, K, N) in enumerate(LAYERS):
        Wt = make_weight(N, K, 11 + i)
        W[("pt", name)] = per_channel(Wt)
        W[("bw", name)] = per_block(Wt)
        if name == "gate_up":
            # the fused gate_up + SiLU*mul quant reads [gate j | up j] 128-row blocks
            qb, sbk = W[("bw", name)]
            W[("bw", name)] = (fq.interleave_gate_up(qb.view(torch.uint8)).view(torch.float8_e4m3fn),
                               fq.interleave_gate_up(sbk, block=1))
        if not args.no_e8m0:
            q8, s8 = per_block(Wt, pow2=True)
            W[("e8", name)] = (q8, (torch.log2(s8).round() + 127).to(torch.uint8).contiguous())
        del Wt

    # ---- activation buffers and workspaces, per scheme
    def scheme_buffers(sc):
        gm = sc != "pt"                      # group-major 1x128 scales
        sdt = torch.uint8 if sc == "e8" else torch.float32

        def sc_buf(L):
            return torch.empty((L // 128, M) if gm else (M, 1), dtype=sdt, device=dev)

        b = {"qa": torch.empty((M, H), dtype=f8, device=dev), "sa": sc_buf(H),
             "yqkv": torch.empty((M, QKV), dtype=torch.bfloat16, device=dev),
             "qo": torch.empty((M, ATT), dtype=f8, device=dev), "so": sc_buf(ATT),
             "h1": torch.empty((M, H), dtype=torch.bfloat16, device=dev),
             "qm": torch.empty((M, H), dtype=f8, device=dev), "sm": sc_buf(H),
             "gu": (torch.empty((M, 2 * I), dtype=torch.bfloat16, device=dev) if sc != "bw" else None),
             "qh": torch.empty((M, I), dtype=f8, device=dev), "sh": sc_buf(I),
             "out": torch.empty((M, H), dtype=torch.bfloat16, device=dev)}
        mode = {"pt": False, "bw": True, "e8": 2}[sc]
        b["ws"] = {name: fq.make_workspace(M, N, K, mode, dev) for name, K, N in LAYERS}
        return b

    schemes = ["pt", "bw"] + ([] if args.no_e8m0 else ["e8"])
    B = {sc: scheme_buffers(sc) for sc in schemes}
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def chain(sc, xin, ain, out=None):
        """The launches of one scheme's stack: list of (name, kind, units, fn)."""
        b = B[sc]
        out = b["out"] if out is None else out
        ue = {"pt": False, "bw": False, "e8": "packed"}[sc]
        lay = "row_major" if sc == "pt" else "group_major"
        gs = (lambda L: L) if sc == "pt" else (lambda L: 128)
        tag = {"pt": "per-token", "bw": "1x128", "e8": "1x128 e8m0"}[sc]

        def gemm(name, a, sa, y):
            Wq, Ws = W[(sc, name)]
            ws = b["ws"][name]
            if sc == "pt":
                return lambda: fq.fp8q_scaled_mm(a, Wq, sa.view(-1), Ws, y=y, workspace=ws)
            if sc == "bw":
                return lambda: fq.fp8q_scaled_mm_blockwise(a, Wq, sa, Ws, a_scale_layout="group_major",
                                                           y=y, workspace=ws)
            return lambda: fq.fp8q_scaled_mm_blockwise_e8m0(a, Wq, sa, Ws, a_scale_layout="group_major",
                                                            y=y, workspace=ws)

        gname = {"pt": "scaled_mm", "bw": "scaled_mm_blockwise", "e8": "scaled_mm_blockwise_e8m0"}[sc]
        fl = {name: 2 * M * N * K for name, K, N in LAYERS}
        return [
            (f"rmsnorm_quant {tag} (H={H})", "quant", quant_bytes("rmsnorm_quant", M, H, gs(H)),
             lambda: fq.fp8q_rmsnorm_quant(xin, w_in, EPS, gs(H), ue, q=b["qa"], scales=b["sa"],
                                           scale_layout=lay)),
            (f"{gname} qkv ({M}x{QKV}x{H})", "gemm", fl["qkv"], gemm("qkv", b["qa"], b["sa"], b["yqkv"])),
            (f"group_quant {tag} (K={ATT})", "quant", quant_bytes("group_quant", M, ATT, gs(ATT)),
             lambda: fq.fp8q_group_quant(ain, gs(ATT), ue, q=b["qo"], scales=b["so"], scale_layout=lay)),
            (f"{gname} o ({M}x{H}x{ATT})", "gemm", fl["o"], gemm("o", b["qo"], b["so"], b["h1"])),
            (f"rmsnorm_quant {tag} (H={H}, o output)", "quant", quant_bytes("rmsnorm_quant", M, H, gs(H)),
             lambda: fq.fp8q_rmsnorm_quant(b["h1"], w_post, EPS, gs(H), ue, q=b["qm"], scales=b["sm"],
                                           scale_layout=lay)),
        ] + ([
            (f"scaled_mm_blockwise_silu_quant gate_up+silu*mul quant 1x128 ({M}x{2 * I}x{H})", "gemm",
             fl["gate_up"],
             lambda: fq.fp8q_scaled_mm_blockwise_silu_quant(
                 b["qm"], W[(sc, "gate_up")][0], b["sm"], W[(sc, "gate_up")][1],
                 a_scale_layout="group_major", q=b["qh"], scales=b["sh"], scale_layout="group_major")),
        ] if sc == "bw" else [
            (f"{gname} gate_up ({M}x{2 * I}x{H})", "gemm", fl["gate_up"],
             gemm("gate_up", b["qm"], b["sm"], b["gu"])),
            (f"silu_mul_quant {tag} (I={I})", "quant", quant_bytes("silu_mul_quant", M, I, gs(I)),
             lambda: fq.fp8q_silu_mul_quant(b["gu"], gs(I), ue, q=b["qh"], scales=b["sh"],
                                            scale_layout=lay)),
        ]) + [
            (f"{gname} down ({M}x{H}x{I})", "gemm", fl["down"], gemm("down", b["qh"], b["sh"], out)),
        ]

    launches = chain("pt", x, attn) + chain("bw", x, attn)
    LAUNCHES_PER_STEP = len(launches)

    def run_step(ls, evs=None):
        for j, (_, _, _, fn) in enumerate(ls):
            fn()
            if evs is not None:
                evs[j].record(stream)

    # ---- warm-up
    for _ in range(args.warmup):
        run_step(launches)
    torch.cuda.synchronize()
    st = fq.fp8q_last_device_status()
    if st != fq.OK:
        raise RuntimeError(f"device status after warm-up: {fq.fp8q_status_string(st)}")

    def barrier():
        if world > 1:
            dist.barrier()

    def timed(ls, steps, sampler=None):
        """Per step: untimed L2 flush, start event, every launch followed by an
        event.  Returns (step times, per-launch times), ms."""
        ev = lambda: torch.cuda.Event(enable_timing=True)
        starts = [ev() for _ in range(steps)]
        per = [[ev() for _ in ls] for _ in range(steps)]
        barrier()
        torch.cuda.synchronize()
        if sampler:
            sampler.start()
        for i in range(steps):
            flush.zero_()
            starts[i].record(stream)
            run_step(ls, per[i])
        torch.cuda.synchronize()
        clocks = sampler.stop() if sampler else None
        barrier()
        step_ms = [s.elapsed_time(p[-1]) for s, p in zip(starts, per)]
        launch_ms = [[(starts[i] if j == 0 else per[i][j - 1]).elapsed_time(per[i][j])
                      for i in range(steps)] for j in range(len(ls))]
        return step_ms, launch_ms, clocks

    # ---- timed: device-resident inputs
    sampler = ClockSampler(local_rank)
    step_ms, launch_ms, clocks = timed(launches, args.steps, sampler)
    total_ms = sum(step_ms)

    # ---- timed: end to end through host buffers (see the module docstring)
    NBUF = 2
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    xd = [(torch.empty_like(x), torch.empty_like(attn)) for _ in range(NBUF)]
    yd = [(torch.empty((M, H), dtype=torch.bfloat16, device=dev),
           torch.empty((M, H), dtype=torch.bfloat16, device=dev)) for _ in range(NBUF)]
    e2e_launches = [chain("pt", xd[b][0], xd[b][1], yd[b][0]) + chain("bw", xd[b][0], xd[b][1], yd[b][1])
                    for b in range(NBUF)]
    out_pinned = [torch.empty((2, M, H), dtype=torch.bfloat16).pin_memory() for _ in range(NBUF)]
    evn = lambda: torch.cuda.Event(enable_timing=False)
    in_done = [evn() for _ in range(args.steps)]
    comp_done = [evn() for _ in range(args.steps)]
    out_done = [evn() for _ in range(args.steps)]
    e_start = torch.cuda.Event(enable_timing=True)
    e_end = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e_start.record(stream)
    s_in.wait_stream(stream)
    s_out.wait_stream(stream)
    for i in range(args.steps):
        b = i % NBUF
        with torch.cuda.stream(s_in):
            if i >= NBUF:
                s_in.wait_event(comp_done[i - NBUF])       # step i-2 has read xd[b]
            xd[b][0].copy_(x_pinned, non_blocking=True)
            xd[b][1].copy_(a_pinned, non_blocking=True)
            in_done[i].record(s_in)
        stream.wait_event(in_done[i])
        if i >= NBUF:
            stream.wait_event(out_done[i - NBUF])          # yd[b] has reached the host
        flush.zero_()
        run_step(e2e_launches[b])
        comp_done[i].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(comp_done[i])
            out_pinned[b][0].copy_(yd[b][0], non_blocking=True)
            out_pinned[b][1].copy_(yd[b][1], non_blocking=True)
            out_done[i].record(s_out)
    stream.wait_event(out_done[args.steps - 1])
    e_end.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = e_start.elapsed_time(e_end)

    # ---- the E8M0 chain (blockwise stack with packed UE8M0 scales), timed alone
    e8 = None
    if not args.no_e8m0:
        l8 = chain("e8", x, attn)
        for _ in range(max(1, args.warmup)):
            run_step(l8)
        s8, lm8, _ = timed(l8, args.steps)
        e8 = (l8, s8, lm8)
    # ---- fused_qk_norm_rope on the step's qkv output (the attention-side op of
    # the same forward pass; not part of the quant+GEMM metric), timed alone
    rope = None
    if not args.no_rope:
        hq, hk, hv, hd = 64, 8, 8, 128
        qkv = B["pt"]["yqkv"]
        cs = torch.randn((32768, hd), device=dev)
        pos = torch.randint(0, 32768, (M,), dtype=torch.int64, device=dev)
        qw = (1.0 + 0.1 * torch.randn(hd, device=dev)).to(torch.bfloat16)
        kw = (1.0 + 0.1 * torch.randn(hd, device=dev)).to(torch.bfloat16)
        rl = [(f"qk_norm_rope neox (T={M}, {hq}+{hk} heads of {hd})", "quant",
               M * (hq + hk) * hd * 2 * 2 + M * (hd * 4 + 8),
               lambda: fq.fp8q_qk_norm_rope(qkv, hq, hk, hv, hd, EPS, qw, kw, cs, pos, True))]
        for _ in range(max(1, args.warmup)):
            run_step(rl)
        _, lmr, _ = timed(rl, args.steps)
        rope = (rl, lmr)
    st = fq.fp8q_last_device_status()
    if st != fq.OK:
        raise RuntimeError(f"device status after timing: {fq.fp8q_status_string(st)}")

    # ---- max over ranks
    total_ms, e2e_ms = max_over_ranks([total_ms, e2e_ms], world, dev)

    flops_step = gemm_flops(M)
    value = job_tflops(flops_step, args.steps, world, total_ms)
    e2e_value = job_tflops(flops_step, args.steps, world, e2e_ms)
    peaks = load_peaks()
    peak, peak_src = fp8_peak(peaks, total_ms * 1e-3)
    hbm = peaks.get("hbm_gbs")
    hbm_src = "of measured: copy bandwidth" if hbm else "of fallback: 6.65 TB/s"
    hbm = hbm or 6650.0

    def kernel_rows(ls, lms):
        gemms, quants = [], []
        for (name, kind, units, _), ms in zip(ls, lms):
            avg_s = statistics.mean(ms) * 1e-3
            if kind == "gemm":
                a = units / avg_s / 1e12
                gemms.append({"kernel": name, "us": round(avg_s * 1e6, 1), "bound": "tensor",
                              "achieved": round(a, 1), "peak": round(peak, 1), "unit": "TFLOP/s",
                              "frac": round(a / peak, 4), "flops": units})
            else:
                a = units / avg_s / 1e9
                quants.append({"kernel": name, "us": round(avg_s * 1e6, 1), "bound": "hbm",
                               "achieved": round(a, 1), "peak": round(hbm, 1), "unit": "GB/s",
                               "frac": round(a / hbm, 4), "bytes": units})
        return gemms, quants

    gemms, quants = kernel_rows(launches, launch_ms)
    share = [statistics.mean(ms) for ms in launch_ms]
    dom = max(range(len(launches)), key=lambda j: share[j])
    dname, dkind, dunits, _ = launches[dom]
    davg = share[dom] * 1e-3
    if dkind == "gemm":
        roof = {"bound": "tensor", "kernel": dname, "achieved": round(dunits / davg / 1e12, 1),
                "peak": round(peak, 1), "unit": "TFLOP/s", "frac": round(dunits / davg / 1e12 / peak, 4),
                "peak_source": peak_src,
                "frac_of_nominal_fp8": round(dunits / davg / 1e12 / NOMINAL_FP8_TFLOPS, 4)}
    else:
        roof = {"bound": "hbm", "kernel": dname, "achieved": round(dunits / davg / 1e9, 1),
                "peak": round(hbm, 1), "unit": "GB/s", "frac": round(dunits / davg / 1e9 / hbm, 4),
                "peak_source": hbm_src}
    roof["share_of_step"] = round(share[dom] / (sum(share)), 4)
    cap = TRAFFIC_CAPTURES.get((dname.split(" ")[0], M))
    if cap and gemm_sources_digest() == cap["sources_sha256"]:
        roof["traffic"] = cap["read"] + cap["write"]
        roof["traffic_note"] = (f"ncu dram__bytes_read.sum {cap['read']} + dram__bytes_write.sum "
                                f"{cap['write']} of one full-size launch of this kernel build (not "
                                f"measured in this run); algorithmic bytes {fused_gate_up_bytes(M)}")
    else:
        roof["traffic"] = None
        roof["traffic_note"] = ("no ncu capture of this kernel build at this size; DRAM bytes of the "
                                "captured builds are in the profiles")

    line = {
        "metric": METRIC,
        "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "e4m3",
        "data": "synthetic (seeded Student-t(3) activations with outlier channels, N(0,1) attention "
                "output stand-in, N(0,0.02) weights)",
        "config": workload_config(M, world),
        "gpu_launches": LAUNCHES_PER_STEP * args.steps,
        "e2e": {"value": round(e2e_value, 2), "unit": "TFLOP/s",
                "h2d_bytes_per_step": (x.numel() + attn.numel()) * 2,
                "d2h_bytes_per_step": 2 * M * H * 2,
                "ms_per_step": round(e2e_ms / args.steps, 4),
                "copies": "pinned host buffers, own streams, double-buffered against the "
                          "neighbouring steps' kernels; L2 flush inside the timed region"},
        "roofline": roof,
        "gemms": gemms,
        "roofline_quant": quants,
        "clocks": clocks,
    }
    if clocks:
        line["clocks"]["time_x_sm_mhz"] = round(total_ms / args.steps * clocks["sm_mhz"], 1)
    if rope is not None:
        _, qr = kernel_rows(*rope)
        line["qk_norm_rope"] = qr[0]
        line["qk_norm_rope"]["bytes_note"] = ("q and k heads read and written once, the token's "
                                              "cos/sin row and position read once")
        line["gpu_launches"] += args.steps
    if e8 is not None:
        l8, s8, lm8 = e8
        g8, q8 = kernel_rows(l8, lm8)
        t8 = sum(s8)
        f8_step = sum(2 * M * N * K for _, K, N in LAYERS)
        line["e8m0_chain"] = {
            "what": "the blockwise stack with packed UE8M0 (E8M0 byte) scales: fused quant ops with "
                    "ue8m0='packed' -> scaled_mm_blockwise_e8m0 (block-scaled tcgen05 MMA)",
            "ms_per_step": round(t8 / args.steps, 4),
            "value": round(f8_step * args.steps / (t8 * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
            "gemms": g8, "roofline_quant": q8}
        line["gpu_launches"] += len(l8) * args.steps
    return line


# ------------------------------------------------------------------ oracle arm
def run_reference(args):
    """The CPU oracle, as it stands, on a bounded sample of the same workload:
    every op of the step on `rows` tokens (weights: seeded random e4m3 codes
    with random scales -- the oracle's cost does not depend on the values)."""
    import numpy as np

    import fp8q_inputs as inp
    import oracle

    M = args.m
    rows = int(os.environ.get("FP8Q_REF_ROWS", "8"))
    x = inp.heavy_tailed_bf16(2000, rows, H)
    att = inp.normal_bf16(2100, (rows, ATT))
    w_in, w_post = inp.rms_weight_bf16(2001, H), inp.rms_weight_bf16(2002, H)
    Wq = {name: inp.random_e4m3_codes_u8(31 + i, (N, K)) for i, (name, K, N) in enumerate(LAYERS)}
    s_ch = {name: inp.random_scales(41 + i, (N,)) for i, (name, K, N) in enumerate(LAYERS)}
    s_bl = {name: inp.random_scales(51 + i, (N // 128, K // 128)) for i, (name, K, N) in enumerate(LAYERS)}

    def stack(g, mm):
        qa, sa = oracle.rmsnorm_quant(x, w_in, EPS, g(H))
        mm("qkv", qa, sa)
        qo, so = oracle.group_quant(att, g(ATT))
        h1 = inp.to_bf16_bits(mm("o", qo, so))
        qm, sm = oracle.rmsnorm_quant(h1, w_post, EPS, g(H))
        gu = inp.to_bf16_bits(mm("gate_up", qm, sm))
        qh, sh = oracle.silu_mul_quant(gu, g(I))
        mm("down", qh, sh)

    def step():
        stack(lambda L: L,
              lambda n, a, s: oracle.scaled_mm(a, Wq[n], s.reshape(-1), s_ch[n])[0])
        stack(lambda L: 128,
              lambda n, a, s: oracle.scaled_mm_blockwise(a, Wq[n], s, s_bl[n])[0])

    for _ in range(max(1, min(args.warmup, 1))):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    value = gemm_flops(rows) * args.steps / dt / 1e12
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    sample = (f"{rows} of {M} tokens per step (every op of the step on those tokens; "
              f"value = their GEMM FLOPs / oracle time)")
    return {
        "metric": METRIC,
        "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(M, 1), "impl": "reference",
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def cpu_baseline_leg(args):
    """Oracle timed on a bounded sample (rank 0, N=1 only)."""
    os.environ.setdefault("FP8Q_REF_ROWS", "32")
    a = argparse.Namespace(**vars(args))
    a.steps, a.warmup = 1, 0
    r = run_reference(a)
    return {"value": r["value"], "unit": "TFLOP/s", "cores": r["cpu_baseline"]["cores"],
            "kind": "oracle", "sample": r["cpu_baseline"]["sample"] + ", 1 step"}


# ------------------------------------------------------------------ per-op sweep
def run_oracle_sweep(args):
    """The CPU oracle, as it stands, per op on the config shapes, on every host
    core and on one core (one child process each, OMP_NUM_THREADS set before the
    oracle library loads).  Quant ops run on their full shapes; GEMMs on the
    full shape for M <= 128 and on a 64-row slice above, extrapolated linearly
    in M (marked "extrapolated").  One JSON line per case."""
    if os.environ.get("FP8Q_ORACLE_SWEEP_CHILD") != "1":
        for threads in (os.cpu_count() or 1, 1):
            env = dict(os.environ, OMP_NUM_THREADS=str(threads), OPENBLAS_NUM_THREADS=str(threads),
                       FP8Q_ORACLE_SWEEP_CHILD="1")
            r = subprocess.run([sys.executable, os.path.abspath(__file__), "--sweep", "oracle"],
                               env=env, stdout=sys.stdout, stderr=sys.stderr)
            if r.returncode != 0:
                return r.returncode
        return 0

    import numpy as np

    import fp8q_inputs as inp
    import oracle

    threads = int(os.environ["OMP_NUM_THREADS"])

    def timed(fn):
        t0 = time.perf_counter()
        fn()
        return time.perf_counter() - t0

    def emit(d):
        d.update({"impl": "oracle", "threads": threads})
        print(json.dumps(d), flush=True)

    w = {h: inp.rms_weight_bf16(2001, h) for h in (4096, 5120)}
    for M in (2048, 8192):
        for op, L in (("group_quant", 4096), ("rmsnorm_quant", 4096), ("rmsnorm_quant", 5120),
                      ("silu_mul_quant", 12288), ("silu_mul_quant", 25600)):
            x = inp.heavy_tailed_bf16(3000 + L, M, 2 * L if op == "silu_mul_quant" else L)
            for g in (L, 128):
                if op == "group_quant":
                    t = timed(lambda: oracle.group_quant(x, g))
                    nbytes = M * (2 * L + L + 4 * (L // g))
                elif op == "rmsnorm_quant":
                    t = timed(lambda: oracle.rmsnorm_quant(x, w[L], EPS, g))
                    nbytes = M * (2 * L + L + 4 * (L // g)) + 2 * L
                else:
                    t = timed(lambda: oracle.silu_mul_quant(x, g))
                    nbytes = M * (4 * L + L + 4 * (L // g))
                emit({"op": op, "M": M, "L": L, "group": g, "s": round(t, 4),
                      "GB/s": round(nbytes / t / 1e9, 3)})
            del x

    s8, s32 = inp.linear_shapes(inp.QWEN3_8B), inp.linear_shapes(inp.QWEN3_32B)
    cases = ([("qwen3-8b", s8, L, M, False) for L in ("gate_up", "down") for M in (1, 16, 128, 2048)]
             + [("qwen3-8b", s8, L, M, True) for L in ("qkv", "o", "gate_up", "down")
                for M in (1, 128, 2048)]
             + [("qwen3-32b", s32, L, 1, True) for L in ("qkv", "o", "gate_up", "down")]
             + [("qwen3-32b", s32, L, 8192, bw) for bw in (False, True)
                for L in ("qkv", "o", "gate_up", "down")])
    for model, sh, layer, M, bw in cases:
        K, N = sh[layer]
        rows = min(M, 64)
        a = inp.random_e4m3_codes(11, (rows, K))
        b = inp.random_e4m3_codes(12, (N, K))
        if bw:
            sa, sb = inp.random_scales(13, (rows, K // 128)), inp.random_scales(14, (N // 128, K // 128))
            t = timed(lambda: oracle.scaled_mm_blockwise(a, b, sa, sb))
        else:
            sa, sb = inp.random_scales(13, (rows,)), inp.random_scales(14, (N,))
            t = timed(lambda: oracle.scaled_mm(a, b, sa, sb))
        t *= M / rows
        emit({"op": "scaled_mm_blockwise" if bw else "scaled_mm", "shape": f"{model} {layer}",
              "M": M, "N": N, "K": K, "s": round(t, 4),
              "TFLOP/s": round(2.0 * M * N * K / t / 1e12, 6), "extrapolated": rows < M,
              "rows_timed": rows})
        del a, b
    return 0


def run_sweep(args):
    """Time every op of the path on the config shapes, one JSON line per case:
    device time per launch (CUDA events, median of --reps, L2 flushed before each
    rep), achieved GB/s or TFLOP/s and the fraction of the measured peak.  Small
    batches (quant M <= 128, GEMM M <= 64) are also replayed from a CUDA graph and
    their per-call time reported (GEMM weights rotated across copies > L2)."""
    import numpy as np
    import torch

    import fp8_quantized_linear_rms_b200 as fq
    import fp8q_inputs as inp

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peaks = {}
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            peaks = json.load(f)
    except Exception:
        pass
    hbm = peaks.get("hbm_gbs", 6650.0)
    fp8_peak = 2.0 * peaks.get("bf16_tflops", 1590.0)      # burst: kernels timed alone
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def sweep_ms(default):
        return tuple(int(v) for v in args.sweep_m.split(",")) if args.sweep_m else default

    def timeit(fn):
        fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(args.reps):
            flush.zero_()
            # keep the GPU busy while the host enqueues fn, so that host-side
            # launch overhead does not leak into the device time of fn
            torch.cuda._sleep(200_000)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            b.synchronize()
            ts.append(a.elapsed_time(b) * 1e-3)
        assert fq.fp8q_last_device_status() == fq.OK
        return float(np.median(ts))

    def graph_time(fns):
        """Per-call device time of fns[0], fns[1], ... replayed back to back
        from one CUDA graph (median over --reps replays)."""
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            for f in fns:
                f()
        stream.wait_stream(side)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for f in fns:
                f()
        g.replay()
        torch.cuda.synchronize()
        ts = []
        for _ in range(args.reps):
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            g.replay()
            b.record(stream)
            b.synchronize()
            ts.append(a.elapsed_time(b) * 1e-3 / len(fns))
        assert fq.fp8q_last_device_status() == fq.OK
        del g
        return float(np.median(ts))

    def emit(d):
        print(json.dumps(d), flush=True)

    def bf16_rand(shape, seed, heavy=True):
        g = torch.Generator(device=dev).manual_seed(seed)
        x = torch.randn(shape, generator=g, device=dev)
        if heavy:
            x = x * (1.0 + 19.0 * (torch.rand(shape[-1], generator=g, device=dev) < 0.01))
        return x.to(torch.bfloat16)

    which = args.sweep
    if which in ("quant", "all"):
        w = {h: bf16_rand((h,), 1, False) * 0.1 + 1.0 for h in (4096, 5120)}
        for M in sweep_ms((16, 128, 2048, 8192)):
            cases = [("group_quant", 4096), ("rmsnorm_quant", 4096), ("rmsnorm_quant", 5120),
                     ("silu_mul_quant", 12288), ("silu_mul_quant", 25600)]
            for op, L in cases:
                for g in (L, 128):
                    if op == "silu_mul_quant":
                        x = bf16_rand((M, 2 * L), 3)
                        fn = lambda: fq.fp8q_silu_mul_quant(x, g)
                        nbytes = M * (4 * L + L + 4 * (L // g))
                    elif op == "rmsnorm_quant":
                        x = bf16_rand((M, L), 4)
                        fn = lambda: fq.fp8q_rmsnorm_quant(x, w[L], 1e-6, g)
                        nbytes = M * (2 * L + L + 4 * (L // g)) + 2 * L
                    else:
                        x = bf16_rand((M, L), 5)
                        fn = lambda: fq.fp8q_group_quant(x, g)
                        nbytes = M * (2 * L + L + 4 * (L // g))
                    t = timeit(fn)
                    d = {"op": op, "M": M, "L": L, "group": g, "us": round(t * 1e6, 2),
                         "GB/s": round(nbytes / t / 1e9, 1),
                         "frac_hbm": round(nbytes / t / 1e9 / hbm, 3)}
                    if M <= 128:
                        # small batches: 16 calls replayed from a CUDA graph (input L2-resident)
                        d["graph_us_per_call"] = round(graph_time([fn] * 16) * 1e6, 2)
                    emit(d)
                    del x

    def gemm_case(tag, M, N, K, blockwise):
        """blockwise: False (scaled_mm), True (fp32 block scales), "e8m0" (E8M0 block
        scales, block-scaled MMA) or "i8" (W8A8_INT8)."""
        scheme = {False: 0, True: 1, "e8m0": 2, "i8": 3}[blockwise]
        if scheme == 3:
            a = torch.randint(-128, 128, (M, K), dtype=torch.int8, device=dev)
            b = torch.randint(-128, 128, (N, K), dtype=torch.int8, device=dev)
        else:
            a = torch.randint(0, 126, (M, K), dtype=torch.uint8, device=dev).view(torch.float8_e4m3fn)
            b = torch.randint(0, 126, (N, K), dtype=torch.uint8, device=dev).view(torch.float8_e4m3fn)
        ws = fq.make_workspace(M, N, K, scheme, dev)
        if scheme == 1:
            sa = torch.rand((K // 128, M), device=dev) * 1e-3 + 1e-4
            sb = torch.rand((N // 128, K // 128), device=dev) * 1e-3 + 1e-4
            call = lambda bb: fq.fp8q_scaled_mm_blockwise(a, bb, sa, sb, a_scale_layout="group_major",
                                                          workspace=ws)
        elif scheme == 2:
            sa = torch.randint(110, 130, (K // 128, M), dtype=torch.uint8, device=dev)
            sb = torch.randint(110, 130, (N // 128, K // 128), dtype=torch.uint8, device=dev)
            call = lambda bb: fq.fp8q_scaled_mm_blockwise_e8m0(a, bb, sa, sb, a_scale_layout="group_major",
                                                               workspace=ws)
        else:
            sa = torch.rand(M, device=dev) * 1e-3 + 1e-4
            sb = torch.rand(N, device=dev) * 1e-3 + 1e-4
            mm = fq.fp8q_scaled_mm_i8 if scheme == 3 else fq.fp8q_scaled_mm
            call = lambda bb: mm(a, bb, sa, sb, workspace=ws)
        fn = lambda: call(b)
        t = timeit(fn)
        flops = 2.0 * M * N * K
        nbytes = M * K + N * K + 2 * M * N
        v = fq.fp8q_select_gemm_variant(M, N, K, scheme)
        op = ["scaled_mm", "scaled_mm_blockwise", "scaled_mm_blockwise_e8m0", "scaled_mm_i8"][scheme]
        d = {"op": op, "shape": tag, "M": M,
             "N": N, "K": K, "variant": v, "us": round(t * 1e6, 2),
             "TFLOP/s": round(flops / t / 1e12, 1), "frac_fp8_peak": round(flops / t / 1e12 / fp8_peak, 3),
             "GB/s": round(nbytes / t / 1e9, 1), "frac_hbm": round(nbytes / t / 1e9 / hbm, 3)}
        if M <= 64:
            # weight streaming: one CUDA graph replays a call on each of enough
            # copies of the weights (384 MiB in all) that every call reads its
            # weights from HBM, as a model's successive layers do
            copies = max(2, min(64, -(-(384 << 20) // (N * K))))
            bs = [b] + [torch.empty_like(b).copy_(b) for _ in range(copies - 1)]
            fns = [lambda bb=bb: call(bb) for bb in bs]
            tg = graph_time(fns)
            d.update({"graph_us_per_call": round(tg * 1e6, 2),
                      "graph_GB/s": round(nbytes / tg / 1e9, 1),
                      "graph_frac_hbm": round(nbytes / tg / 1e9 / hbm, 3)})
            del bs, fns
        emit(d)

    if which in ("gemm8b", "all"):
        sh = inp.linear_shapes(inp.QWEN3_8B)
        for M in sweep_ms((1, 16, 128, 2048)):
            for layer in ("gate_up", "down"):
                K, N = sh[layer]
                gemm_case(f"qwen3-8b {layer}", M, N, K, False)
        for M in sweep_ms((1, 2, 4, 8, 16, 32, 64, 128, 256, 512, 1024, 2048, 4096)):
            for layer in ("qkv", "o", "gate_up", "down"):
                K, N = sh[layer]
                gemm_case(f"qwen3-8b {layer}", M, N, K, True)
    if which in ("decode32b", "all"):
        sh = inp.linear_shapes(inp.QWEN3_32B)
        for M in sweep_ms((1, 2, 4, 8, 16, 32, 64)):
            for layer in ("qkv", "o", "gate_up", "down"):
                K, N = sh[layer]
                gemm_case(f"qwen3-32b {layer}", M, N, K, True)
    def fused_gate_up_case(tag, M, K, N2):
        """The gate_up GEMM with the SiLU*mul 1x128 quant in its epilogue, on the
        bench step's kind of operands (heavy-tailed activations normalized and
        quantized in 1x128 groups, N(0, 0.02) weights in 128x128 blocks), beside
        the plain blockwise GEMM of the same operands (bf16 [gate | up] out)."""
        x = bf16_rand((M, K), 5)
        w = torch.ones(K, device=dev, dtype=torch.bfloat16)
        a, sa = fq.fp8q_rmsnorm_quant(x, w, 1e-6, 128, scale_layout="group_major")
        g = torch.Generator(device=dev).manual_seed(6)
        wb = (torch.randn(N2, K, generator=g, device=dev) * 0.02).view(N2 // 128, 128, K // 128, 128)
        sb = wb.abs().amax(dim=(1, 3)).clamp_min(1e-10) / 448.0
        b = (wb / sb[:, None, :, None]).clamp(-448, 448).to(torch.float8_e4m3fn).view(N2, K)
        b = fq.interleave_gate_up(b.view(torch.uint8)).view(torch.float8_e4m3fn)
        sb = fq.interleave_gate_up(sb.contiguous(), block=1)
        del wb, x
        q = torch.empty((M, N2 // 2), dtype=torch.float8_e4m3fn, device=dev)
        s = torch.empty((N2 // 256, M), dtype=torch.float32, device=dev)
        y = torch.empty((M, N2), dtype=torch.bfloat16, device=dev)
        flops = 2.0 * M * N2 * K
        t_sq = timeit(lambda: fq.fp8q_scaled_mm_blockwise_silu_quant(a, b, sa, sb, a_scale_layout="group_major",
                                                                      q=q, scales=s, scale_layout="group_major"))
        t_bw = timeit(lambda: fq.fp8q_scaled_mm_blockwise(a, b, sa, sb, a_scale_layout="group_major", y=y))
        emit({"op": "scaled_mm_blockwise_silu_quant", "shape": tag, "M": M, "N": N2, "K": K,
              "fused_quant": "exact" if fq.fp8q_get_fused_quant_exact() else "fast",
              "us": round(t_sq * 1e6, 2), "TFLOP/s": round(flops / t_sq / 1e12, 1),
              "frac_fp8_peak": round(flops / t_sq / 1e12 / fp8_peak, 3),
              "plain_blockwise_us": round(t_bw * 1e6, 2), "fused_over_plain": round(t_sq / t_bw, 3)})

    def library_case(tag, M, N, K, scales):
        """torch's FP8 GEMM (torch._scaled_mm / F.scaled_mm) on the same shape, as
        the measured library figure beside this library's: row-wise scales (per
        token x per channel), one scale per tensor, or 1x128 x 128x128 blocks."""
        a = torch.randint(0, 126, (M, K), dtype=torch.uint8, device=dev).view(torch.float8_e4m3fn)
        b = torch.randint(0, 126, (N, K), dtype=torch.uint8, device=dev).view(torch.float8_e4m3fn)
        if scales == "blockwise":
            # 1x128 activation groups, 128x128 weight blocks, in the layouts the
            # library takes: [M, K/128] and [K/128, N/128], both M-/K-block-major
            import torch.nn.functional as F
            sa = (torch.rand((K // 128, M), device=dev) * 1e-3 + 1e-4).t()
            sb = (torch.rand((N // 128, K // 128), device=dev) * 1e-3 + 1e-4).t()
            fn = lambda: F.scaled_mm(a, b.t(), sa, F.ScalingType.BlockWise1x128, sb,
                                     F.ScalingType.BlockWise128x128, output_dtype=torch.bfloat16)
        elif scales == "rowwise":
            sa = torch.rand((M, 1), device=dev) * 1e-3 + 1e-4
            sb = torch.rand((1, N), device=dev) * 1e-3 + 1e-4
            fn = lambda: torch._scaled_mm(a, b.t(), scale_a=sa, scale_b=sb, out_dtype=torch.bfloat16)
        else:
            sa = torch.tensor(1e-3, device=dev)
            sb = torch.tensor(1e-3, device=dev)
            fn = lambda: torch._scaled_mm(a, b.t(), scale_a=sa, scale_b=sb, out_dtype=torch.bfloat16)
        d = {"op": "torch._scaled_mm", "scales": scales, "shape": tag, "M": M, "N": N, "K": K}
        try:
            t = timeit(fn)
        except Exception as e:                      # a scaling the installed library lacks
            d["unavailable"] = f"{type(e).__name__}: {str(e)[:160]}"
            emit(d)
            return
        flops = 2.0 * M * N * K
        d.update({"us": round(t * 1e6, 2), "TFLOP/s": round(flops / t / 1e12, 1),
                  "frac_fp8_peak": round(flops / t / 1e12 / fp8_peak, 3)})
        emit(d)

    if which in ("library", "all"):
        sh = inp.linear_shapes(inp.QWEN3_32B)
        for scales in ("rowwise", "tensor", "blockwise"):
            for layer in ("qkv", "o", "gate_up", "down"):
                K, N = sh[layer]
                library_case(f"qwen3-32b {layer}", 8192, N, K, scales)

    if which in ("prefill32b", "all"):
        sh = inp.linear_shapes(inp.QWEN3_32B)
        for bw in (False, True, "e8m0", "i8"):
            for layer in ("qkv", "o", "gate_up", "down"):
                K, N = sh[layer]
                gemm_case(f"qwen3-32b {layer}", 8192, N, K, bw)
        K, N2 = sh["gate_up"]
        fused_gate_up_case("qwen3-32b gate_up", 8192, K, N2)
        fq.fp8q_set_fused_quant_exact(True)
        fused_gate_up_case("qwen3-32b gate_up", 8192, K, N2)
        fq.fp8q_set_fused_quant_exact(False)
    if which in ("e8m0", "all"):
        sh8, sh32 = inp.linear_shapes(inp.QWEN3_8B), inp.linear_shapes(inp.QWEN3_32B)
        for M in sweep_ms((1, 16, 64, 256, 1024, 4096)):
            for layer in ("qkv", "o", "gate_up", "down"):
                K, N = sh8[layer]
                gemm_case(f"qwen3-8b {layer}", M, N, K, "e8m0")
        for M in (1, 8, 64):
            for layer in ("qkv", "o", "gate_up", "down"):
                K, N = sh32[layer]
                gemm_case(f"qwen3-32b {layer}", M, N, K, "e8m0")
    return 0


def main():
    args = parse()
    os.environ.setdefault("OMP_NUM_THREADS", str(os.cpu_count() or 1))
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.sweep == "oracle":
        return run_oracle_sweep(args)
    if args.sweep:
        return run_sweep(args)
    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args)), flush=True)
        return 0
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    line = run_native(args, rank, world, local_rank)
    if rank == 0:
        if world == 1:
            line["cpu_baseline"] = cpu_baseline_leg(args)
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
