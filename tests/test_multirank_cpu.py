"""The multi-rank host logic of bench.py on CPU: two gloo ranks on 127.0.0.1.

Under torchrun every rank runs its own replica of the batch (no collective on
the data path); the job's time is the slowest rank's, taken by an all-reduce
MAX, and the whole-job throughput counts every rank's tokens.  The reference
arm runs on rank 0 only: other ranks return at once, without work.
"""
import datetime
import os
import socket
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class _RefArgs:
    steps, warmup, gpus = 1, 0, 2


def _rank_main(rank, world, port, times_ms, out):
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import torch.distributed as dist

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = bench.max_over_ranks(times_ms[rank], "cpu")
        tok = bench.job_tokens_per_s(16, 10, world, ms)
        ref = bench.run_reference(_RefArgs()) if rank != 0 else "skipped"   # rank 0 would run the oracle
        dist.barrier()
    finally:
        dist.destroy_process_group()
    out.put((rank, ms, tok, ref))


def test_two_gloo_ranks_take_the_slowest_time_and_sum_the_tokens():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    times = [12.5, 20.0]
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, times, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, tok, ref in res:
        assert ms == 20.0                                  # the slowest rank's time, on every rank
        assert tok == 16 * 10 * 2 / 0.020                  # both ranks' tokens over that time
    assert res[1][3] is None                               # reference arm: rank 1 returns without work


def test_single_rank_helpers_without_a_process_group():
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(7.0, "cpu") == 7.0
    assert bench.job_tokens_per_s(16, 256, 1, 1000.0) == 16 * 256
