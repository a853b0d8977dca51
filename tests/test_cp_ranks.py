"""The multi-rank plumbing of context-parallel decode on CPU (gloo, two
ranks): the token ranges every rank derives, and the all-gather that stacks
the ranks' partials in rank order.  The compute steps are CUDA kernels and
are covered on one GPU by tests/test_gpu_cp.py."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from long_context_decode_flash_b200 import cp, flint


def test_rank_ranges_cover_the_context_in_order():
    for L, world in [(1, 1), (7, 2), (262_144, 8), (100_001, 3), (9, 9)]:
        rr = cp.rank_ranges(L, world)
        assert rr[0][0] == 0 and rr[-1][1] == L
        assert all(a[1] == b[0] for a, b in zip(rr, rr[1:]))
        sizes = [hi - lo for lo, hi in rr]
        assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1
    with pytest.raises(ValueError):
        cp.rank_ranges(3, 4)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        B = 3
        part = torch.full((B, flint.CP_PARTIAL_FLOATS), float(rank), dtype=torch.float32)
        part[:, 0] = torch.arange(B, dtype=torch.float32) + 10 * rank
        got = cp.gather_partials(part)
        ok = tuple(got.shape) == (world, B, flint.CP_PARTIAL_FLOATS)
        for r in range(world):
            ok = ok and bool((got[r, :, 1:] == r).all()) and got[r, :, 0].tolist() == [10 * r, 10 * r + 1, 10 * r + 2]
        q.put((rank, ok))
    finally:
        dist.destroy_process_group()


def test_gather_stacks_partials_in_rank_order_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert results == {0: True, 1: True}
