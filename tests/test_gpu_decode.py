"""Parity of flint_attn_decode (split-KV flash-decode with sinks) against the
float64 oracle, through the C ABI, on seeded inputs."""
import numpy as np
import pytest
import torch

import oracle
from long_context_decode_flash_b200 import flint
from long_context_decode_flash_b200 import inputs as I

from helpers import check_workspace_clean, dev, parity

pytestmark = pytest.mark.gpu


def run_decode(q, k, v, seq_lens, sinks, window, layout=flint.CONTIGUOUS, capacity=0,
               table=None, num_blocks=0, num_ctas=0, req_stride=0):
    cache = flint.kv_cache(k, v, layout, capacity=capacity, block_table=table,
                           num_blocks=num_blocks, req_stride=req_stride)
    B = len(seq_lens)
    out = torch.full((B, 32, 128), float("nan"), dtype=torch.float32, device="cuda")
    ws = flint.workspace(B, num_ctas)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    flint.flint_attn_decode(q, cache, seq_lens, sinks, window, out, ws, num_ctas=num_ctas,
                            dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    check_workspace_clean(ws)  # ready for the next call
    return out.cpu().numpy()


def oracle_contig(d: I.DecodeInputs, b, window, sinks=None):
    s = d.sinks.numpy().astype(np.float64) if sinks is None else sinks
    return oracle.attn_decode(I.bits(d.q[b]), I.bits(d.k_cache[b]), I.bits(d.v_cache[b]),
                              d.seq_lens[b], s, window)


@pytest.mark.parametrize("L", [1, 2, 63, 64, 65, 127, 500, 512, 513, 514, 1000, 2048, 5000])
@pytest.mark.parametrize("window", [0, 513])
def test_contiguous_single_request(L, window):
    d = I.make_decode(L, workload=I.W_FULL_SMALL, capacity=L + 37)
    got = run_decode(dev(d.q), dev(d.k_cache), dev(d.v_cache), d.seq_lens, dev(d.sinks), window,
                     capacity=L + 37)
    parity(got[0], oracle_contig(d, 0, window), f"L={L} window={window}")


def test_full_layer_2048_fp32_q_and_split_counts():
    """Small full layer (context 2048): q as bf16 and as fp32, many split counts;
    results agree with the oracle and with one another."""
    d = I.make_decode(2048, workload=I.W_FULL_SMALL)
    want = oracle_contig(d, 0, 0)
    k, v, s = dev(d.k_cache), dev(d.v_cache), dev(d.sinks)
    outs = []
    for q in (dev(d.q), dev(d.q.float())):
        for n in (0, 1, 3, 7, 64, 148):
            got = run_decode(q, k, v, d.seq_lens, s, 0, capacity=2048, num_ctas=n)
            parity(got[0], want, f"num_ctas={n}")
            outs.append(got)
    # the same split count gives the same bits for bf16 q and its exact fp32
    # copy; other split counts reorder fp32 sums and the bf16 hi/lo split of P
    for a in outs[1:6]:
        np.testing.assert_allclose(a, outs[0], rtol=1e-4, atol=1e-5)
    for a, b in zip(outs[:6], outs[6:]):
        assert np.array_equal(a, b)


def test_deterministic_run_to_run():
    d = I.make_decode(20000, workload=I.W_FULL_SMALL)
    args = (dev(d.q), dev(d.k_cache), dev(d.v_cache), d.seq_lens, dev(d.sinks), 0)
    a = run_decode(*args, capacity=20000)
    b = run_decode(*args, capacity=20000)
    assert np.array_equal(a, b)


def test_workspace_reused_across_plans():
    """One workspace through calls of different plans: a problem merged a CTA
    per unit (9,000 tokens over every SM), one merged a warp per unit, a
    ragged batch, a launch with no merge at the end, and the first call again.
    The items' ready flags carry the launch count, so a flag left by an
    earlier plan never passes for a new one: every call matches the oracle,
    a repeated call gives the same bits, and the workspace is left clean."""
    ws = flint.workspace(3)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    big = I.make_decode(9000, workload=I.W_FULL_SMALL + 40)
    small = I.make_decode(2048, workload=I.W_FULL_SMALL + 41)
    batch = I.make_decode(5000, workload=I.W_FULL_SMALL + 42, B=3)
    batch.seq_lens = [5000, 700, 3000]
    want_big, want_small = oracle_contig(big, 0, 0), oracle_contig(small, 0, 0)
    want_batch = [oracle_contig(batch, b, 0) for b in range(3)]

    def call(d, num_ctas=0):
        cache = flint.kv_cache(dev(d.k_cache), dev(d.v_cache), flint.CONTIGUOUS,
                               capacity=d.k_cache.shape[1])
        out = torch.full((len(d.seq_lens), 32, 128), float("nan"), dtype=torch.float32, device="cuda")
        flint.flint_attn_decode(dev(d.q), cache, d.seq_lens, dev(d.sinks), 0, out, ws,
                                num_ctas=num_ctas, dev_err=err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        check_workspace_clean(ws)
        return out.cpu().numpy()

    first = call(big)
    parity(first[0], want_big, "9000 tokens, first call")
    for n in (148, 0):
        parity(call(small, n)[0], want_small, f"2048 tokens, num_ctas={n}")
    got = call(batch)
    for b in range(3):
        parity(got[b], want_batch[b], f"batch request {b}")
    parity(call(small, 7)[0], want_small, "2048 tokens on 7 CTAs (merged inline)")
    again = call(big)
    assert np.array_equal(again, first)


def test_full_layer_100k_matches_oracle():
    """Full NoPE layer at context 100,000 (205 MB of KV), every head, in the
    launch configuration the benchmark uses."""
    d = I.make_decode(100_000, workload=I.W_FULL_100K)
    got = run_decode(dev(d.q), dev(d.k_cache), dev(d.v_cache), d.seq_lens, dev(d.sinks), 0,
                     capacity=100_000)
    parity(got[0], oracle_contig(d, 0, 0), "L=100000")


def test_sinks_to_minus_infinity_and_large():
    d = I.make_decode(3000, workload=I.W_FULL_SMALL)
    for sinks in (np.full(32, -np.inf), np.full(32, 30.0), np.linspace(-20, 20, 32)):
        s = torch.tensor(sinks, dtype=torch.float32)
        got = run_decode(dev(d.q), dev(d.k_cache), dev(d.v_cache), d.seq_lens, dev(s), 0,
                         capacity=3000)
        want = oracle_contig(d, 0, 0, sinks.astype(np.float32).astype(np.float64))
        if np.isinf(sinks).any():
            parity(got[0], want, "sink -inf")
        else:
            # a dominant sink shrinks the output: compare in absolute terms
            assert np.abs(got[0] - want).max() <= 2e-3
            assert np.linalg.norm(got[0] - want) <= 1e-3 * np.linalg.norm(want) + 1e-9


def test_garbage_beyond_the_context_is_ignored():
    """Slots past the context hold NaN: masked rows must not leak into the output."""
    L, cap = 1000, 1100
    d = I.make_decode(L, workload=I.W_FULL_SMALL, capacity=cap)
    k, v = dev(d.k_cache), dev(d.v_cache)
    k.view(torch.int16)[:, L:] = 0x7fc0
    v.view(torch.int16)[:, L:] = 0x7fc0
    for window in (0, 513):
        got = run_decode(dev(d.q), k, v, d.seq_lens, dev(d.sinks), window, capacity=cap)
        parity(got[0], oracle_contig(d, 0, window), f"window={window}")


def test_batched_contiguous_ragged_lengths_with_stride():
    lens = [1, 77, 4096, 513, 9000]
    cap = 9100
    B = len(lens)
    q = I.bf16_normal((B, 32, 128), 123)
    # requests 9216 slots apart: a padded request stride
    stride_tok = 9216
    kc = I.bf16_normal((B, stride_tok, 4, 128), 124)
    vc = I.bf16_normal((B, stride_tok, 4, 128), 125)
    sinks = I.f32_normal((32,), 126)
    for window in (0, 513):
        got = run_decode(dev(q), dev(kc), dev(vc), lens, dev(sinks), window, capacity=cap,
                         req_stride=stride_tok * 512)
        for b, L in enumerate(lens):
            want = oracle.attn_decode(I.bits(q[b]), I.bits(kc[b]), I.bits(vc[b]), L,
                                      sinks.numpy().astype(np.float64), window)
            parity(got[b], want, f"b={b} L={L} window={window}")


@pytest.mark.parametrize("L", [600, 5000, 513 * 64 + 7])
def test_ring_cache(L):
    lay = I.make_layer(I.W_SWA_100K, 1, L, 513, True, ring=True)
    q = I.bf16_normal((1, 32, 128), 77)
    got = run_decode(dev(q), dev(lay.k_cache)[None], dev(lay.v_cache)[None], [L], dev(lay.sinks),
                     513, layout=flint.RING, capacity=513)
    want = oracle.attn_decode(I.bits(q[0]), I.bits(lay.k_cache), I.bits(lay.v_cache), L,
                              lay.sinks.numpy().astype(np.float64), 513, layout=oracle.RING,
                              capacity=513)
    parity(got[0], want, f"ring L={L}")


def test_ring_cache_short_context():
    # fewer than 513 positions: only slots 0..L-1 are valid
    L = 200
    lay = I.make_layer(I.W_SWA_100K, 2, L, 513, True, ring=True)
    k, v = dev(lay.k_cache), dev(lay.v_cache)
    k.view(torch.int16)[L:] = 0x7fc0
    v.view(torch.int16)[L:] = 0x7fc0
    q = I.bf16_normal((1, 32, 128), 78)
    got = run_decode(dev(q), k[None], v[None], [L], dev(lay.sinks), 513, layout=flint.RING,
                     capacity=513)
    want = oracle.attn_decode(I.bits(q[0]), I.bits(lay.k_cache), I.bits(lay.v_cache), L,
                              lay.sinks.numpy().astype(np.float64), 513, layout=oracle.RING,
                              capacity=513)
    parity(got[0], want, "ring short")


@pytest.mark.parametrize("window", [0, 513])
def test_paged_small_batch(window):
    pb = I.make_paged_batch(seq_lens=[1, 64, 65, 700, 3000, 130], spare_blocks=9,
                            workload=I.W_PAGED_BATCH)
    nb = pb.k_pool.shape[0]
    got = run_decode(dev(pb.q), dev(pb.k_pool), dev(pb.v_pool), pb.seq_lens, dev(pb.sinks), window,
                     layout=flint.PAGED, table=dev(pb.block_table), num_blocks=nb)
    for b, L in enumerate(pb.seq_lens):
        want = oracle.attn_decode(I.bits(pb.q[b]), I.bits(pb.k_pool), I.bits(pb.v_pool), L,
                                  pb.sinks.numpy().astype(np.float64), window, layout=oracle.PAGED,
                                  block_table=pb.block_table[b].numpy(), block_size=64)
        parity(got[b], want, f"paged b={b} L={L} window={window}")


def test_paged_equals_contiguous_bitwise_shape():
    """A permuted block table over the same rows gives the same result as the
    contiguous cache (same plan shape), up to fp32 reassociation."""
    L = 4000
    d = I.make_decode(L, workload=I.W_FULL_SMALL, capacity=4032)
    nb = 4032 // 64
    perm = torch.randperm(nb, generator=torch.Generator().manual_seed(4)).to(torch.int32)
    kp = torch.empty((nb, 64, 4, 128), dtype=torch.bfloat16)
    vp = torch.empty_like(kp)
    kp[perm.long()] = d.k_cache[0].reshape(nb, 64, 4, 128)
    vp[perm.long()] = d.v_cache[0].reshape(nb, 64, 4, 128)
    a = run_decode(dev(d.q), dev(d.k_cache), dev(d.v_cache), [L], dev(d.sinks), 0, capacity=4032)
    b = run_decode(dev(d.q), dev(kp), dev(vp), [L], dev(d.sinks), 0, layout=flint.PAGED,
                   table=dev(perm[None]), num_blocks=nb)
    np.testing.assert_allclose(a, b, rtol=1e-4, atol=1e-5)


def test_paged_block_id_out_of_range_sets_device_error():
    pb = I.make_paged_batch(seq_lens=[300], workload=I.W_PAGED_BATCH)
    table = pb.block_table.clone()
    # a block id beyond the pool: the tiles of that block are never loaded (no
    # coordinate outside the tensor reaches TMA), the error is flagged, and the
    # output is meaningless
    table[0, 2] = pb.k_pool.shape[0] + 5
    cache = flint.kv_cache(dev(pb.k_pool), dev(pb.v_pool), flint.PAGED, block_table=dev(table),
                           num_blocks=pb.k_pool.shape[0])
    out = torch.empty((1, 32, 128), dtype=torch.float32, device="cuda")
    ws = flint.workspace(1)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    flint.flint_attn_decode(dev(pb.q), cache, [300], dev(pb.sinks), 0, out, ws, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == flint.FLINT_ERR_INVALID_ARG


def test_workspace_too_small_is_rejected():
    d = I.make_decode(100, workload=I.W_FULL_SMALL)
    cache = flint.kv_cache(dev(d.k_cache), dev(d.v_cache), flint.CONTIGUOUS, capacity=100)
    out = torch.empty((1, 32, 128), dtype=torch.float32, device="cuda")
    ws = torch.zeros(64, dtype=torch.uint8, device="cuda")
    with pytest.raises(flint.FlintError) as e:
        flint.flint_attn_decode(dev(d.q), cache, [100], dev(d.sinks), 0, out, ws)
    assert e.value.status == flint.FLINT_ERR_WORKSPACE
