"""Time every GEMM variant on this GPU and write the library's variant table.

    python -m fp8_quantized_linear_rms_b200.tune [--out FILE] [--json FILE] [--reps N]

For each scheme (per-token/per-channel scales, 1x128/128x128 block scales),
each linear-layer shape (N, K) of the Qwen3-8B and Qwen3-32B models and each
bucket of M, every candidate variant -- Swap-AB or not, tile width, whole-K
tiles, split-K factors, stream-K, CTA pairs -- is timed on the device, and the fastest
goes into ``csrc/fp8q_variant_table.inc``, which ``fp8q_gemm.cu`` compiles in.
Rebuild the library afterwards (``python fp8_quantized_linear_rms_b200/build.py``).

Timing: CUDA events around a run of back-to-back calls, each on its own copy
of the weight matrix, with enough copies (384 MiB in all, 2 to 64 of them) that every
call reads its weights from HBM as a model's successive layers do; the time
per call is the median over trials of the run's mean.  Each trial times every
candidate once, in an order rotated from trial to trial, so that the GPU's
clock under its power cap drifts over all candidates alike.

Where variants come within 2% of the fastest, the simplest wins, in this
order: whole-K tiles, split-K, stream-K (they need no / a fixed / a larger
workspace).  Operands are random e4m3 codes and positive scales; the time of a
variant does not depend on the values.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import re
import statistics

import torch

import fp8_quantized_linear_rms_b200 as fq

HERE = os.path.dirname(os.path.abspath(__file__))

# (name, K, N) of the linear layers: Qwen3-8B (hidden 4096, intermediate 12288,
# 32 query / 8 kv heads of 128), Qwen3-32B (hidden 5120, intermediate 25600,
# 64 query / 8 kv heads of 128), and a square 2048 layer.
SHAPES = [
    ("qwen3-8b qkv", 4096, 6144), ("qwen3-8b o", 4096, 4096),
    ("qwen3-8b gate_up", 4096, 24576), ("qwen3-8b down", 12288, 4096),
    ("qwen3-32b qkv", 5120, 10240), ("qwen3-32b o", 8192, 5120),
    ("qwen3-32b gate_up", 5120, 51200), ("qwen3-32b down", 25600, 5120),
    ("square 2048", 2048, 2048),
]
M_BUCKETS = [1, 8, 16, 32, 64, 128, 256, 512, 1024, 2048, 4096, 8192]
DECODE_MAX_M = 8
TIE = 1.02


def _tiles(rows_a: int, rows_b: int, bn: int) -> int:
    return -(-rows_a // 128) * -(-rows_b // bn)


def _effective_split(s: int, kblocks: int) -> int:
    """Split factor the library runs for a requested s: ceil(kblocks / s) K blocks
    per split, so only ceil(kblocks / that) splits are non-empty."""
    per = -(-kblocks // s)
    return -(-kblocks // per)


def _splits(tiles: int, kblocks: int, sms: int) -> list[int]:
    out = [1]
    if tiles < 2 * sms:
        out.append(0)                       # stream-K
    if tiles < sms:
        fit = sms // tiles
        for s in sorted({2, 3, 4, 6, 8, fit}):
            if 1 < s <= min(fit, kblocks):
                e = _effective_split(s, kblocks)
                if e > 1 and e not in out:
                    out.append(e)
    return out


def candidates(M: int, N: int, K: int, sms: int, blockwise: bool) -> list[tuple[int, int, int, int]]:
    """(swap_ab, split_k, block_n, cta_pair) variants worth timing for this shape."""
    kb = K // 128
    out = []
    if M <= DECODE_MAX_M and K % 128 == 0 and N % 16 == 0:
        out.append((1, 1, 8, 0))            # warp-MMA weight streaming
    if M <= 128:
        bn = next(b for b in (16, 32, 64, 128) if b >= M)
        for b in sorted({bn, min(128, 2 * bn)}):
            out += [(1, s, b, 0) for s in _splits(_tiles(N, M, b), kb, sms)]
    if M >= 32:
        for b in (128, 256):
            out += [(0, s, b, 0) for s in _splits(_tiles(M, N, b), kb, sms)]
    if M >= 256 and not blockwise:
        # CTA pairs: 256x256 tiles on two SMs.  (The blockwise pair kernel,
        # whose two CTAs hand every K block's partial back and forth, and
        # 128-wide pairs never come near the single-CTA variants.)
        out += [(0, 1, 256, 1)]
    return out


def _complexity(v):
    return 0 if v[1] == 1 else (1 if v[1] > 1 else 2)


def _time_run(fns, trials: int) -> float:
    """Mean time per call (us) of calling fns[0], fns[1], ... back to back."""
    for f in fns:
        f()
    torch.cuda.synchronize()
    per = []
    for _ in range(trials):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        # The GPU sleeps while the host queues the run, so host-side call
        # overhead never leaves the GPU idle between the timed calls.
        torch.cuda._sleep(50_000 * len(fns))
        a.record()
        for f in fns:
            f()
        b.record()
        b.synchronize()
        per.append(a.elapsed_time(b) * 1e3 / len(fns))
    return statistics.median(per)


def _round_robin(runs, reps: int, time_one) -> dict:
    """Median over `reps` trials of time_one(v, fns) for every (v, fns) in runs.
    Trial r goes round the candidates starting at candidate r mod len(runs), so
    that every candidate is timed at every point of the GPU's warming under its
    power cap (timing one candidate's trials after another's let the later one
    run at a lower clock)."""
    per = {v: [] for v, _ in runs}
    for r in range(reps):
        k = r % len(runs)
        for v, fns in runs[k:] + runs[:k]:
            per[v].append(time_one(v, fns))
    return {v: statistics.median(ts) for v, ts in per.items()}


def tune(reps: int = 5, shapes=SHAPES, buckets=M_BUCKETS, log=print):
    dev = torch.device("cuda", torch.cuda.current_device())
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    rows = []
    for name, K, N in shapes:
        copies = max(2, min(64, -(-(384 << 20) // (N * K))))
        bs = [torch.randint(0, 0x7E, (N, K), dtype=torch.uint8, device=dev, generator=g)
              .view(torch.float8_e4m3fn) for _ in range(copies)]
        sb_ch = torch.rand(N, device=dev, generator=g) * 1e-3
        sb_bl = torch.rand((N // 128, K // 128), device=dev, generator=g) * 1e-3
        for M in buckets:
            a = torch.randint(0, 0x7E, (M, K), dtype=torch.uint8, device=dev, generator=g)
            a = a.view(torch.float8_e4m3fn)
            sa_tok = torch.rand(M, device=dev, generator=g) * 1e-3
            sa_grp = torch.rand((K // 128, M), device=dev, generator=g) * 1e-3
            y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            for bw in (0, 1):
                # Each candidate's calls, with the workspace its variant needs.
                runs = []
                for v in candidates(M, N, K, sms, bool(bw)):
                    fq.fp8q_force_gemm_variant(*v)
                    try:
                        ws = fq.make_workspace(M, N, K, bool(bw), dev)
                    finally:
                        fq.fp8q_force_gemm_variant()
                    if bw:
                        fns = [lambda b=b, ws=ws: fq.fp8q_scaled_mm_blockwise(
                            a, b, sa_grp, sb_bl, a_scale_layout="group_major", y=y,
                            workspace=ws) for b in bs]
                    else:
                        fns = [lambda b=b, ws=ws: fq.fp8q_scaled_mm(a, b, sa_tok, sb_ch, y=y,
                                                                    workspace=ws) for b in bs]
                    runs.append((v, fns))

                def time_one(v, fns):
                    fq.fp8q_force_gemm_variant(*v)
                    try:
                        return _time_run(fns, 1)
                    finally:
                        fq.fp8q_force_gemm_variant()

                times = _round_robin(runs, reps, time_one)
                del runs
                best_t = min(times.values())
                best = min((v for v, t in times.items() if t <= best_t * TIE),
                           key=lambda v: (_complexity(v), times[v]))
                row = {"shape": name, "blockwise": bw, "m_max": M, "N": N, "K": K,
                       "variant": list(best), "us": round(times[best], 2),
                       "tflops": round(2.0 * M * N * K / times[best] / 1e6, 1),
                       "all": {",".join(map(str, v)): round(t, 2) for v, t in times.items()}}
                rows.append(row)
                log(json.dumps(row))
            del a, y
        del bs
    return rows


_ROW = re.compile(r"^\{(\d+), (\d+), (\d+), (\d+), (\d+), (\d+), (\d+), (\d+)\},\s*// (.*?): ([0-9.]+) us$")


def merge_rows(rows, path: str):
    """The table at `path` with the measured rows replacing (or joining) those of
    the same (scheme, m_max, N, K); returns row dicts in shape, scheme, M order."""
    have = {}
    with open(path) as f:
        for line in f:
            m = _ROW.match(line.strip())
            if m:
                v = [int(x) for x in m.groups()[:8]]
                have[(v[0], v[1], v[2], v[3])] = {"shape": m.group(9), "blockwise": v[0], "m_max": v[1],
                                                  "N": v[2], "K": v[3], "variant": v[4:8],
                                                  "us": float(m.group(10))}
    for r in rows:
        have[(r["blockwise"], r["m_max"], r["N"], r["K"])] = r
    order = {name: i for i, (name, _, _) in enumerate(SHAPES)}
    return sorted(have.values(), key=lambda r: (order.get(r["shape"], 99), r["m_max"], r["blockwise"]))


def write_table(rows, path: str, device: str | None = None) -> None:
    dev = device or torch.cuda.get_device_name()
    with open(path, "w") as f:
        f.write(f"// Measured GEMM variant table, written by tune.py on {dev}\n")
        f.write(f"// ({datetime.date.today().isoformat()}): the fastest variant per scheme, (N, K)\n")
        f.write("// and bucket of M (mean microseconds per call, weights read from HBM).\n")
        f.write("// {blockwise, m_max, N, K, swap_ab, split_k (0 = stream-K), block_n, cta_pair}\n")
        for r in rows:
            s, k, n, c = r["variant"]
            f.write(f"{{{r['blockwise']}, {r['m_max']}, {r['N']}, {r['K']}, {s}, {k}, {n}, {c}}},"
                    f"  // {r['shape']}: {r['us']} us\n")


def main():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--out", default=os.path.join(HERE, "csrc", "fp8q_variant_table.inc"))
    ap.add_argument("--json", default=None, help="also write every timing as JSON lines")
    ap.add_argument("--reps", type=int, default=5, help="trials per variant")
    ap.add_argument("--buckets", default=None,
                    help="comma-separated M buckets to measure (default: all); the measured rows "
                         "replace those of the same buckets in the existing table, the others stay")
    args = ap.parse_args()
    jf = open(args.json, "w") if args.json else None

    def log(line):
        print(line, flush=True)
        if jf:
            jf.write(line + "\n")
            jf.flush()

    if args.buckets:
        rows = tune(args.reps, buckets=[int(b) for b in args.buckets.split(",")], log=log)
        rows = merge_rows(rows, args.out)
    else:
        rows = tune(args.reps, log=log)
    write_table(rows, args.out)
    if jf:
        jf.close()


if __name__ == "__main__":
    main()
