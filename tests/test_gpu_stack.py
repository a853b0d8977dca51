"""Parity of flint_attn_stack (one token through the 49-layer attention stack
in one launch: per-head Q/K RMSNorm, RoPE on window layers, KV append, split
decode with sinks) against the float64 oracle, layer by layer."""
import numpy as np
import pytest
import torch

import oracle
from long_context_decode_flash_b200 import flint
from long_context_decode_flash_b200 import inputs as I

from helpers import DeviceLayer, bf16_ulp_diff, dev, oracle_layer, parity, stack_on_gpu

pytestmark = pytest.mark.gpu


def check_layer(lay, got, dl, what):
    want, kc, vc = oracle_layer(lay)
    parity(got, want, what)
    k_dev = I.bits(dl.k_cache.cpu())
    v_dev = I.bits(dl.v_cache.cpu())
    # v is copied bit for bit; k agrees with the oracle's rounding within 1 ulp
    assert np.array_equal(v_dev, vc), f"{what}: v cache differs"
    d = bf16_ulp_diff(k_dev, kc)
    assert d.max() <= 1, f"{what}: k cache differs by {d.max()} ulps"
    changed = np.argwhere((k_dev != I.bits(lay.k_cache)).any(axis=(1, 2))).ravel()
    slot = (lay.L - 1) % lay.capacity if lay.layout == flint.RING else lay.L - 1
    assert set(changed.tolist()) <= {slot}, f"{what}: rows {changed} written"


@pytest.mark.parametrize("L", [1, 100, 513, 514, 3000])
def test_stack_small_context(L):
    layers = I.make_stack(L, workload=I.W_STACK_100K + 10)
    got, dls = stack_on_gpu(layers, L - 1)
    for i, (lay, dl) in enumerate(zip(layers, dls)):
        check_layer(lay, got[i], dl, f"L={L} layer {i}")


def test_stack_split_invariance_and_determinism():
    L = 7000
    layers = I.make_stack(L, workload=I.W_STACK_100K + 11)
    outs = []
    for n in (0, 0, 13, 148):
        got, _ = stack_on_gpu(layers, L - 1, num_ctas=n)
        outs.append(got)
    assert np.array_equal(outs[0], outs[1])
    # another split count moves where P is rounded to its bf16 hi/lo parts and
    # reorders fp32 sums: agreement to ~1e-5 relative, far inside the parity bar
    for o in outs[2:]:
        np.testing.assert_allclose(o, outs[0], rtol=1e-4, atol=1e-5)


def test_stack_workspace_sizes_agree_with_the_oracle():
    """The run-time queue is sized by the workspace: the full workspace, the
    no-alloc scratch's 251 partials and the static-plan minimum (no queue) give
    three different plans; each agrees with the oracle, and with the others to
    rounding."""
    L = 20_000
    layers = I.make_stack(L, workload=I.W_STACK_100K + 12)
    dl = [DeviceLayer(l) for l in layers]
    arr = flint.stack_layers(dl)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    G = 148
    outs = []
    for items in (768, 251, G + 49):
        ws = torch.zeros(4096 + items * 16640, dtype=torch.uint8, device="cuda")
        out = torch.full((49, 32, 128), float("nan"), dtype=torch.float32, device="cuda")
        flint.flint_attn_stack(arr, L - 1, out, ws, num_ctas=G, dev_err=err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        outs.append(out.cpu().numpy())
    kinds = I.layer_kinds()
    full = [i for i, f in enumerate(kinds) if f]
    for o in outs:
        for i in (full[0], full[-1], 0):
            want, _, _ = oracle_layer(layers[i])
            parity(o[i], want, f"layer {i}")
    for o in outs[1:]:
        np.testing.assert_allclose(o, outs[0], rtol=1e-4, atol=1e-5)


def test_stack_100k_sampled_layers():
    """The full 49-layer stack at context 100,000, launched as the benchmark
    launches it; the oracle checks every layer (the full layers' tails are the
    queue's chunks, served by whichever CTA frees up first), every head, and
    the appended rows."""
    L = 100_000
    layers = I.make_stack(L)
    got, dls = stack_on_gpu(layers, L - 1)
    for i in range(len(layers)):
        check_layer(layers[i], got[i], dls[i], f"layer {i}")
    assert np.isfinite(got).all()


def test_single_window_layer_at_100k_two_ways():
    """A sliding-window RoPE layer at context 100,000: through the fused stack
    call with one layer, and through flint_qk_norm_rope (+append) followed by
    flint_attn_decode; both match the oracle."""
    L = 100_000
    lay = I.make_layer(I.W_SWA_100K, 0, L, 513, True, ring=True)
    want, kc, vc = oracle_layer(lay)
    got, dls = stack_on_gpu([lay], L - 1)
    parity(got[0], want, "stack(1)")
    dl = DeviceLayer(lay)
    q_out = torch.empty((1, 32, 128), dtype=torch.float32, device="cuda")
    flint.flint_qk_norm_rope(dl.q_raw[None], dl.k_raw[None], dl.w_q, dl.w_k, [L - 1],
                             apply_rope=True, q_out=q_out, v_raw=dl.v_raw[None], cache=dl.cache)
    out = torch.empty((1, 32, 128), dtype=torch.float32, device="cuda")
    ws = flint.workspace(1)
    cache = flint.kv_cache(dl.k_cache[None], dl.v_cache[None], flint.RING, capacity=513)
    flint.flint_attn_decode(q_out, cache, [L], dl.sinks, 513, out, ws)
    torch.cuda.synchronize()
    parity(out.cpu().numpy()[0], want, "norm_rope+decode")
    assert np.array_equal(I.bits(dl.v_cache.cpu()), vc)
    assert bf16_ulp_diff(I.bits(dl.k_cache.cpu()), kc).max() <= 1
    # both routes append the very same k bits
    assert np.array_equal(I.bits(dl.k_cache.cpu()), I.bits(dls[0].k_cache.cpu()))


def test_stack_with_paged_full_layer():
    """A stack layer may also keep its cache in blocks."""
    L = 5000
    lay = I.make_layer(I.W_STACK_100K + 12, 3, L, 0, False, ring=False)
    nb = -(-L // 64)
    perm = torch.randperm(nb + 3, generator=torch.Generator().manual_seed(8))[:nb].to(torch.int32)
    kp = torch.zeros((nb + 3, 64, 4, 128), dtype=torch.bfloat16)
    vp = torch.zeros_like(kp)
    kflat = torch.zeros((nb * 64, 4, 128), dtype=torch.bfloat16)
    vflat = torch.zeros_like(kflat)
    kflat[:L] = lay.k_cache
    vflat[:L] = lay.v_cache
    kp[perm.long()] = kflat.reshape(nb, 64, 4, 128)
    vp[perm.long()] = vflat.reshape(nb, 64, 4, 128)
    dl = DeviceLayer(lay)
    dl.k_cache, dl.v_cache = dev(kp), dev(vp)
    dl.cache = flint.kv_cache(dl.k_cache, dl.v_cache, flint.PAGED, block_table=dev(perm[None]),
                              num_blocks=nb + 3)
    out = torch.empty((1, 32, 128), dtype=torch.float32, device="cuda")
    ws = flint.workspace(1)
    flint.flint_attn_stack([dl], L - 1, out, ws)
    torch.cuda.synchronize()
    want, kc, vc = oracle_layer(lay)
    parity(out.cpu().numpy()[0], want, "paged stack layer")
    got_k = I.bits(dl.k_cache.cpu())[perm.long().numpy()].reshape(nb * 64, 4, 128)[:L]
    assert bf16_ulp_diff(got_k, kc).max() <= 1
