"""The kernels' time-out path on the GPU, reached without any fault.

Every wait in the decode and prefill kernels is bounded; when one runs out
the kernel sets *dev_err = FLINT_ERR_TIMEOUT, lets its copies in flight land,
and returns.  These tests load a test build of the library
(libflint_hooks.so: the self-checks, a 5 ms wait limit, and hooks that make
one CTA leave one pipeline stage unarmed, so that nothing is ever in flight
for it) and check, per kernel, that the call reports the time-out and ends
within a few wait limits, and that the next call on the same stream (the hook
off, the workspace zeroed as the header asks after a device error) is correct
against the float64 oracle.  The CPU model of this abort path is
tests/test_abort_protocol.py."""
import contextlib
import time

import numpy as np
import pytest
import torch

import oracle
from long_context_decode_flash_b200 import build as cuda_build
from long_context_decode_flash_b200 import flint
from long_context_decode_flash_b200 import inputs as I

from helpers import DeviceLayer, close_bits, dev, oracle_layer, parity, u16

pytestmark = pytest.mark.gpu

LIMIT_S = cuda_build.HOOKS_WAIT_LIMIT_NS * 1e-9


@pytest.fixture(scope="module")
def hooks():
    return flint.open_library(cuda_build.build_hooks())


@contextlib.contextmanager
def using(lib):
    """Route the binding's calls to `lib` for the duration."""
    saved = flint._lib
    flint._lib = lib
    try:
        yield
    finally:
        flint._lib = saved


def timed(fn):
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    fn()
    torch.cuda.synchronize()
    return time.perf_counter() - t0


def test_decode_stack_stalled_stage_times_out_then_recovers(hooks):
    L = 2000
    layers = I.make_stack(L, workload=I.W_STACK_100K + 30)
    dl = [DeviceLayer(l) for l in layers]
    arr = flint.stack_layers(dl)
    out = torch.empty((len(dl), 32, 128), dtype=torch.float32, device="cuda")
    ws = flint.workspace(len(dl))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    with using(hooks):
        assert hooks.flint_test_stall_decode(-1, -1) == 0
        flint.flint_attn_stack(arr, L - 1, out, ws, dev_err=err)  # loads the module, normal run
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        # CTA 5 never arms the stage of its second tile
        assert hooks.flint_test_stall_decode(5, 1) == 0
        dt = timed(lambda: flint.flint_attn_stack(arr, L - 1, out, ws, dev_err=err))
        assert int(err.item()) == flint.FLINT_ERR_TIMEOUT
        # consumers wait one limit, then the drain and the grid barrier at most one each
        assert dt < 6 * LIMIT_S + 0.25, f"the timed-out call took {dt:.3f} s"
        assert hooks.flint_test_stall_decode(-1, -1) == 0
        ws.zero_()
        err.zero_()
        out.fill_(float("nan"))
        flint.flint_attn_stack(arr, L - 1, out, ws, dev_err=err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
    got = out.cpu().numpy()
    kinds = I.layer_kinds()
    for i in (0, kinds.index(True), 48):
        want, _, _ = oracle_layer(layers[i])
        parity(got[i], want, f"layer {i} after a time-out")


def test_decode_full_layer_stalled_stage_times_out_then_recovers(hooks):
    """One problem split over every CTA, merged after the grid barrier: the
    stalled CTA reaches the barrier a wait limit late."""
    L = 9000
    d = I.make_decode(L, workload=I.W_FULL_SMALL + 30)
    q, k, v, sinks = dev(d.q), dev(d.k_cache), dev(d.v_cache), dev(d.sinks)
    cache = flint.kv_cache(k, v, flint.CONTIGUOUS, capacity=L)
    out = torch.empty((1, 32, 128), dtype=torch.float32, device="cuda")
    ws = flint.workspace(1)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    with using(hooks):
        assert hooks.flint_test_stall_decode(-1, -1) == 0
        flint.flint_attn_decode(q, cache, [L], sinks, 0, out, ws, dev_err=err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        assert hooks.flint_test_stall_decode(0, 0) == 0
        dt = timed(lambda: flint.flint_attn_decode(q, cache, [L], sinks, 0, out, ws, dev_err=err))
        assert int(err.item()) == flint.FLINT_ERR_TIMEOUT
        assert dt < 6 * LIMIT_S + 0.25, f"the timed-out call took {dt:.3f} s"
        assert hooks.flint_test_stall_decode(-1, -1) == 0
        ws.zero_()
        err.zero_()
        flint.flint_attn_decode(q, cache, [L], sinks, 0, out, ws, dev_err=err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
    want = oracle.attn_decode(I.bits(d.q[0]), I.bits(d.k_cache[0]), I.bits(d.v_cache[0]), L,
                              d.sinks.numpy().astype(np.float64), 0, capacity=L)
    parity(out.cpu().numpy()[0], want, "full layer after a time-out")


@pytest.mark.parametrize("T,block,tile", [(300, 0, 1), (1000, 147, 5)])
def test_prefill_stalled_k_tile_times_out_then_recovers(hooks, T, block, tile):
    """(300, 0, 1): block 0 holds the last 16 query tokens, three K tiles, and
    the second never arrives.  (1000, 147, 5): 252 units on 148 persistent
    CTAs; CTA 147 walks units 147 and 148 (4 tiles each), and its tile 5, in
    the second unit, never arrives (the CTA has reloaded Q by then)."""
    if torch.cuda.get_device_properties(0).multi_processor_count != 148 and block != 0:
        pytest.skip("the unit deal of this case assumes 148 SMs")
    p = I.make_prefill(T, 0, workload=I.W_PREFILL + 30)
    want, qb, kb = oracle.prefill(I.bits(p.q_raw), I.bits(p.k_raw), I.bits(p.v_raw), I.bits(p.w_q),
                                  I.bits(p.w_k), p.sinks.numpy().astype(np.float64), 0, p.rope,
                                  rows=range(T))
    q = torch.from_numpy(qb.view(np.int16)).view(torch.bfloat16).cuda()
    k = torch.from_numpy(kb.view(np.int16)).view(torch.bfloat16).cuda()
    v16 = dev(p.v_raw.to(torch.float16))
    sinks = dev(p.sinks)
    out = torch.empty((T, 32, 128), dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    with using(hooks):
        assert hooks.flint_test_stall_prefill(-1, -1) == 0
        flint.flint_prefill_attn(q, k, v16, sinks, 0, out, dev_err=err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        assert hooks.flint_test_stall_prefill(block, tile) == 0
        dt = timed(lambda: flint.flint_prefill_attn(q, k, v16, sinks, 0, out, dev_err=err))
        assert int(err.item()) == flint.FLINT_ERR_TIMEOUT
        assert dt < 6 * LIMIT_S + 0.25, f"the timed-out call took {dt:.3f} s"
        assert hooks.flint_test_stall_prefill(-1, -1) == 0
        err.zero_()
        out.fill_(float("nan"))
        flint.flint_prefill_attn(q, k, v16, sinks, 0, out, dev_err=err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
    parity(out.cpu().numpy(), want, "prefill after a time-out", per_head=True)


def test_prefill_prep_stalled_slot_times_out_then_recovers(hooks):
    """The prefill's norm/RoPE pass: CTA 0 leaves the slot of its second token
    unarmed, so its consumer warps' waits run out and its producer, waiting
    for a slot to come free, sees the abort."""
    T = 1000
    p = I.make_prefill(T, flint.WINDOW, workload=I.W_PREFILL + 31)
    _, qb, kb = oracle.prefill(I.bits(p.q_raw), I.bits(p.k_raw), I.bits(p.v_raw), I.bits(p.w_q),
                               I.bits(p.w_k), p.sinks.numpy().astype(np.float64), flint.WINDOW, p.rope, rows=[])
    q_raw, k_raw, v_raw, w_q, w_k = dev(p.q_raw), dev(p.k_raw), dev(p.v_raw), dev(p.w_q), dev(p.w_k)
    q = torch.empty((T, 32, 128), dtype=torch.bfloat16, device="cuda")
    k = torch.empty((T, 4, 128), dtype=torch.bfloat16, device="cuda")
    v16 = torch.empty((T, 4, 128), dtype=torch.float16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")

    def call():
        flint.flint_prefill_qk_norm_rope(q_raw, k_raw, w_q, w_k, apply_rope=p.rope, q_out=q, k_out=k,
                                         v_raw=v_raw, v_out=v16, dev_err=err)

    with using(hooks):
        assert hooks.flint_test_stall_prefill_prep(-1, -1) == 0
        call()
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        assert hooks.flint_test_stall_prefill_prep(0, 1) == 0
        dt = timed(call)
        assert int(err.item()) == flint.FLINT_ERR_TIMEOUT
        assert dt < 6 * LIMIT_S + 0.25, f"the timed-out call took {dt:.3f} s"
        assert hooks.flint_test_stall_prefill_prep(-1, -1) == 0
        err.zero_()
        for t in (q, k, v16):
            t.fill_(float("nan"))
        call()
        torch.cuda.synchronize()
        assert int(err.item()) == 0
    close_bits(u16(q), qb, "q after a time-out")
    close_bits(u16(k), kb, "k after a time-out")
    np.testing.assert_array_equal(u16(v16), u16(p.v_raw.to(torch.float16)))
