"""The multi-GPU host logic of `bench.py`, on the CPU: two ranks over gloo.

The path shards as independent replicas (each rank quantizes and multiplies
its own token batch; there is no data-path collective), so what a multi-rank
launch adds is bookkeeping: every rank takes the element-wise maximum of the
ranks' times (the slowest rank sets the job's time), the job's throughput
counts the FLOPs of all ranks, and the workload names the replicas and the
global batch.
"""
import datetime
import os
import socket
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        # per-rank step time and end-to-end time (ms): rank 1 is slower on the
        # first, rank 0 on the second
        mine = [10.0 + rank, 20.0 - 3.0 * rank]
        total_ms, e2e_ms = bench.max_over_ranks(mine, world)
        flops = bench.gemm_flops(2048)
        q.put((rank, total_ms, e2e_ms, bench.job_tflops(flops, 4, world, total_ms)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_time_the_slowest_rank_and_count_every_ranks_flops():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = {}
    try:
        for _ in range(2):
            rank, total_ms, e2e_ms, tflops = q.get(timeout=180)
            got[rank] = (total_ms, e2e_ms, tflops)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    sys.path.insert(0, ROOT)
    import bench
    flops = bench.gemm_flops(2048)
    # Qwen3-32B block linears, two schemes: 2 x (qkv + o + gate_up + down), 2 M N K each
    H, I = 5120, 25600
    assert flops == 2 * 2 * 2048 * (H * 10240 + 8192 * H + H * 2 * I + I * H)
    for rank in (0, 1):
        total_ms, e2e_ms, tflops = got[rank]
        assert total_ms == 11.0 and e2e_ms == 20.0
        assert abs(tflops - flops * 4 * 2 / 11.0e-3 / 1e12) < 1e-9 * tflops


def test_replica_workload_names_the_global_batch():
    sys.path.insert(0, ROOT)
    import bench
    one, four = bench.workload_config(2048, 1), bench.workload_config(2048, 4)
    assert one["workload"] == four["workload"]       # same per-GPU workload
    assert one["parallelism"] == "single-gpu" and four["parallelism"] == "replicas4"
    assert one["global_batch"] == 2048 and four["global_batch"] == 4 * 2048
    assert four["tokens_per_gpu"] == 2048
