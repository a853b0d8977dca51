"""Context-parallel decode of a full layer on one GPU, its ranks emulated as
separate launches (nothing waits on another rank): every "rank" holds a
contiguous range of the layer's tokens in a cache of its own and runs
flint_attn_decode_partial; the stacked partials go through
flint_merge_partials.  Against the float64 oracle: the merged output equals
the decode attention over the whole context (up to the 262,144-token maximum
context), one rank's partial equals the oracle's attn_partial, and a rank
with no keys merges as nothing."""
import numpy as np
import pytest
import torch

import oracle
from long_context_decode_flash_b200 import cp, flint
from long_context_decode_flash_b200 import inputs as I

from helpers import dev, parity

pytestmark = pytest.mark.gpu

W_CP = 60  # workload ids of their own for the seeded inputs


def rank_partials(q, k, v, ranges, ks=None, vs=None):
    """Each rank's partial over its own tokens: k / v [B, L, 4, 128] on the
    host, split by `ranges` into per-rank device caches."""
    B = q.shape[0]
    parts = torch.empty((len(ranges), B, flint.CP_PARTIAL_FLOATS), dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    for r, (lo, hi) in enumerate(ranges):
        kr, vr = dev(k[:, lo:hi].contiguous()), dev(v[:, lo:hi].contiguous())
        cache = flint.kv_cache(kr, vr, flint.CONTIGUOUS, capacity=hi - lo, k_scale=ks, v_scale=vs)
        flint.flint_attn_decode_partial(q, cache, [hi - lo] * B, parts[r], flint.workspace(B), dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return parts


def merge(parts, sinks):
    out = torch.full((parts.shape[1], 32, 128), float("nan"), dtype=torch.float32, device="cuda")
    flint.flint_merge_partials(parts, sinks, out)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def oracle_full(d, b, L):
    sinks = d.sinks.numpy().astype(np.float64)
    if d.k_scale is not None:
        return oracle.attn_decode_fp8(I.bits(d.q[b]), d.k_cache[b].numpy(), d.v_cache[b].numpy(), d.k_scale,
                                      d.v_scale, L, sinks, 0, capacity=L)
    return oracle.attn_decode(I.bits(d.q[b]), I.bits(d.k_cache[b]), I.bits(d.v_cache[b]), L, sinks, 0, capacity=L)


@pytest.mark.parametrize("L,world", [(5000, 2), (5000, 3), (100_000, 4), (262_144, 8)])
def test_cp_merge_equals_whole_context_decode(L, world):
    d = I.make_decode(L, workload=W_CP)
    parts = rank_partials(dev(d.q), d.k_cache, d.v_cache, cp.rank_ranges(L, world))
    got = merge(parts, dev(d.sinks))
    parity(got[0], oracle_full(d, 0, L), f"L={L} ranks={world}")


def test_cp_batch_uneven_ranges_and_e4m3():
    """Two requests; ranges of 1 token to most of the context; then E4M3 caches."""
    L = 4097
    ranges = [(0, 1), (1, 64), (64, 65), (65, 4000), (4000, L)]
    d = I.make_decode(L, workload=W_CP + 1, B=2)
    got = merge(rank_partials(dev(d.q), d.k_cache, d.v_cache, ranges), dev(d.sinks))
    for b in range(2):
        parity(got[b], oracle_full(d, b, L), f"request {b}")
    d8 = I.make_decode(L, workload=W_CP + 2, fp8=True)
    got8 = merge(rank_partials(dev(d8.q), d8.k_cache, d8.v_cache, ranges, d8.k_scale, d8.v_scale),
                 dev(d8.sinks))
    parity(got8[0], oracle_full(d8, 0, L), "E4M3")


def test_one_rank_partial_matches_the_oracle_partial_and_merges_to_decode():
    L = 3000
    d = I.make_decode(L, workload=W_CP + 3)
    parts = rank_partials(dev(d.q), d.k_cache, d.v_cache, [(0, L)])
    p = parts[0, 0].cpu().numpy().astype(np.float64)
    O, m, lsum = p[:4096].reshape(32, 128), p[4096:4128], p[4128:]
    Ow, mw, lw = oracle.attn_partial(I.bits(d.q[0]), I.bits(d.k_cache[0]), I.bits(d.v_cache[0]))
    # the kernel's reference m is its running maximum, which moves only by
    # steps of more than 8: within 8 below the true maximum
    assert (m <= mw + 1e-3).all() and (m >= mw - 8 - 1e-3).all()
    # the triple is defined up to the common factor 2^m: compare at the oracle's m
    f = np.exp2(m - mw)
    np.testing.assert_allclose(lsum * f, lw, rtol=1e-4)
    parity(O / lsum[:, None], Ow / lw[:, None], "O / l")
    # and the merge of the single partial is flint_attn_decode's output
    out = torch.empty((1, 32, 128), dtype=torch.float32, device="cuda")
    flint.flint_attn_decode(dev(d.q), flint.kv_cache(dev(d.k_cache), dev(d.v_cache), flint.CONTIGUOUS,
                                                     capacity=L), [L], dev(d.sinks), 0, out, flint.workspace(1))
    torch.cuda.synchronize()
    np.testing.assert_allclose(merge(parts, dev(d.sinks))[0], out.cpu().numpy()[0], rtol=1e-5, atol=1e-6)


def test_rank_without_keys_merges_as_nothing():
    L = 2000
    d = I.make_decode(L, workload=W_CP + 4)
    parts = rank_partials(dev(d.q), d.k_cache, d.v_cache, cp.rank_ranges(L, 2))
    empty = torch.zeros((1, 1, flint.CP_PARTIAL_FLOATS), dtype=torch.float32, device="cuda")
    empty[0, 0, 4096:4128] = float("-inf")
    with_empty = torch.cat([parts[:1], empty, parts[1:]])
    np.testing.assert_array_equal(merge(with_empty, dev(d.sinks)), merge(parts, dev(d.sinks)))
    parity(merge(with_empty, dev(d.sinks))[0], oracle_full(d, 0, L), "with an empty rank")


def test_cp_decode_single_process_group_of_one():
    """cp.cp_decode end to end in a process group of one rank (gloo; the
    gather then only stacks): the whole context on this rank."""
    import os
    import socket
    import torch.distributed as dist
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=0, world_size=1)
    try:
        L = 1500
        d = I.make_decode(L, workload=W_CP + 5)
        cache = flint.kv_cache(dev(d.k_cache), dev(d.v_cache), flint.CONTIGUOUS, capacity=L)
        out = torch.empty((1, 32, 128), dtype=torch.float32, device="cuda")
        cp.cp_decode(dev(d.q), cache, [L], dev(d.sinks), out, flint.workspace(1))
        torch.cuda.synchronize()
        parity(out.cpu().numpy()[0], oracle_full(d, 0, L), "cp_decode")
    finally:
        dist.destroy_process_group()


def test_merge_of_only_empty_partials_is_zero_not_nan():
    """Partials with no key at all (m = -inf, l = 0, O = 0), some heads with a
    sink of -inf: the merge has no softmax mass for those heads and gives 0,
    as the oracle's merge does; finite sinks give 0 as well."""
    B = 2
    parts = torch.zeros((3, B, flint.CP_PARTIAL_FLOATS), dtype=torch.float32)
    parts[:, :, 32 * 128:32 * 128 + 32] = float("-inf")
    sinks = torch.randn(32, dtype=torch.float32)
    sinks[::2] = float("-inf")
    got = merge(dev(parts), dev(sinks))
    empty = (np.zeros((32, 128)), np.full(32, -np.inf), np.zeros(32))
    want = oracle.merge_partials([empty] * 3, sinks.numpy().astype(np.float64))
    assert np.isfinite(got).all()
    assert np.array_equal(got[0], want) and np.array_equal(got[1], want)
