"""flint_attn_stack_noalloc, the stack call that runs on the library's own
fixed device scratch instead of a caller's workspace, against flint_attn_stack
on the same inputs.  Two calls in a row on the shared scratch must both agree
with it: the second call starts from what the first one left there.

This file is named so that it is collected after every other test file; it
also passes alone in a fresh process."""
import ctypes

import numpy as np
import pytest
import torch

from long_context_decode_flash_b200 import flint
from long_context_decode_flash_b200 import inputs as I

from helpers import MAX_ABS, REL_L2, DeviceLayer, oracle_layer

WORKLOAD = I.W_STACK_100K + 30


def close(got, want, what):
    got = np.asarray(got, np.float64).reshape(-1, 128)
    want = np.asarray(want, np.float64).reshape(-1, 128)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = np.abs(got - want).max()
    rel = np.linalg.norm(got - want) / np.linalg.norm(want)
    assert err <= MAX_ABS and rel <= REL_L2, f"{what}: max abs {err:.3e}, rel L2 {rel:.3e}"


def run_both(layers, pos, num_ctas=0):
    """flint_attn_stack once with its own workspace, then the no-alloc call twice."""
    dl = [DeviceLayer(l) for l in layers]
    arr = flint.stack_layers(dl)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ref = torch.empty((len(dl), 32, 128), dtype=torch.float32, device="cuda")
    ws = flint.workspace(len(dl), num_ctas)
    flint.flint_attn_stack(arr, pos, ref, ws, num_ctas=num_ctas, dev_err=err)
    outs = []
    for _ in range(2):
        out = torch.full((len(dl), 32, 128), float("nan"), dtype=torch.float32, device="cuda")
        flint.flint_attn_stack_noalloc(arr, pos, out, num_ctas=num_ctas, dev_err=err)
        outs.append(out)
    torch.cuda.synchronize()
    assert int(err.item()) == 0, f"device error {int(err.item())}"
    return ref.cpu().numpy(), [o.cpu().numpy() for o in outs]


@pytest.mark.gpu
def test_noalloc_stack_matches_stack_twice():
    # 49 layers at context 20,000: full layers are split over a few CTAs each
    # and merged by their last-arriving CTA through the scratch counters
    L = 20_000
    layers = I.make_stack(L, workload=WORKLOAD)
    ref, outs = run_both(layers, L - 1)
    for k, o in enumerate(outs):
        close(o, ref, f"call {k + 1}")
    # and against the float64 oracle directly: one full and two window layers
    kinds = I.layer_kinds()
    for i in (kinds.index(True), 0, 48):
        want, _, _ = oracle_layer(layers[i])
        for k, o in enumerate(outs):
            close(o[i], want, f"call {k + 1}, layer {i} against the oracle")


@pytest.mark.gpu
def test_noalloc_grid_merge_matches_stack_twice():
    # one full layer at context 30,000 is split over every CTA and merged after
    # the grid barrier, whose word also lives in the scratch
    L = 30_000
    layers = [I.make_layer(WORKLOAD, 3, L, 0, False, ring=False)]
    for num_ctas in (0, 37):
        ref, outs = run_both(layers, L - 1, num_ctas=num_ctas)
        for k, o in enumerate(outs):
            close(o, ref, f"num_ctas={num_ctas} call {k + 1}")


def min_workspace(n_layers, ctas):
    # the counters plus one partial per static item, at most ctas + n_layers
    return 4096 + (ctas + n_layers) * 16640


def test_noalloc_size_check_counts_the_ctas_launched():
    """The size check counts the CTAs a launch would use: num_ctas, but never
    more than the device has SMs (296, the launch limit, when the count cannot
    be read, as on a machine without a GPU).  Too large a request is refused on
    the host before any device work, with the sizes in the message; one that
    fits goes on to the argument checks (here it is refused for its NULL layer
    pointers)."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count if torch.cuda.is_available() else 296
    need = min_workspace(49, min(296, sms))
    arr = (flint.StackLayer * 49)()
    out = ctypes.c_void_p(16)
    lib = flint.load_library()
    st = lib.flint_attn_stack_noalloc(arr, 49, 0, 1e-6, 1e4, out, 296, None, None)
    msg = lib.flint_last_error().decode()
    if need > 4 << 20:
        assert st == flint.FLINT_ERR_WORKSPACE, msg
        assert str(need) in msg and str(4 << 20) in msg, msg
    else:
        assert st == flint.FLINT_ERR_INVALID_ARG and "NULL" in msg, msg
    # 49 layers on 202 CTAs, the most that fit, pass the size check
    assert min_workspace(49, 202) <= 4 << 20 < min_workspace(49, 203)
