"""The multi-rank host path of bench.py on the CPU: two gloo ranks agree on
the slowest rank's time, and the whole-job figure counts one token per rank
per step (weak scaling, no data-path collective)."""
import datetime
import multiprocessing as mp
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, local_ms, out):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        got = bench.max_over_ranks(local_ms[rank], world, "cpu")
        out.put((rank, got, bench.per_token_us(got, world)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_rank():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    local_ms = [0.41, 0.43]  # rank 1 is the slower one
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, local_ms, out)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        results = sorted(out.get(timeout=120) for _ in procs)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert [p.exitcode for p in procs] == [0, 0]
    for rank, got, per_token in results:
        assert got == pytest.approx(0.43)
        # two tokens per step of the job: 0.43 ms per step -> 215 us per token
        assert per_token == pytest.approx(215.0)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(0.5, 1, "cpu") == 0.5
    assert bench.per_token_us(0.5, 1) == pytest.approx(500.0)


def test_prefill_work_counts_match_brute_force():
    """The prefill roofline's algorithmic work: keys attended summed row by
    row (row t attends min(t + 1, window) keys, or t + 1), 4 x 128 FLOP per
    (row, key, head) over 32 heads."""
    import bench
    for T in (1, 2, 100, 512, 513, 514, 2000, 8192):
        for window in (0, 513):
            brute = sum(min(t + 1, window) if window else t + 1 for t in range(T))
            assert bench.prefill_keys(T, window) == brute
            assert bench.prefill_flops(T, window) == brute * 32 * 128 * 4
    # the 49-layer prompt of the benchmark: 14 full and 35 window layers
    total = 14 * bench.prefill_flops(8192, 0) + 35 * bench.prefill_flops(8192, 513)
    assert total == 10_032_091_496_448
