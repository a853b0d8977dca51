"""flint_attn_layers_serial: the 49-layer stack as 49 serially dependent
launches (programmatic dependent launch), checked against the float64 oracle
layer by layer and against the single-launch stack."""
import numpy as np
import pytest
import torch

from long_context_decode_flash_b200 import flint
from long_context_decode_flash_b200 import inputs as I

from helpers import (DeviceLayer, bf16_ulp_diff, check_workspace_clean, e4m3_code_distance, oracle_layer, parity,
                     stack_on_gpu)

pytestmark = pytest.mark.gpu


def serial_on_gpu(layers, pos, num_ctas=0):
    dl = [DeviceLayer(l) for l in layers]
    out = torch.full((len(dl), 32, 128), float("nan"), dtype=torch.float32, device="cuda")
    ws = flint.workspace(len(dl), num_ctas)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    flint.flint_attn_layers_serial(dl, pos, out, ws, num_ctas=num_ctas, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0, f"device error {int(err.item())}"
    check_workspace_clean(ws)  # the reused workspace is left ready for the next call
    return out.cpu().numpy(), dl


@pytest.mark.parametrize("fp8", [False, True])
def test_serial_stack_matches_the_oracle_every_layer(fp8):
    L = 3000
    layers = I.make_stack(L, workload=I.W_STACK_100K + 50, fp8=fp8)
    got, dls = serial_on_gpu(layers, L - 1)
    for i, (lay, dl) in enumerate(zip(layers, dls)):
        want, kc, vc = oracle_layer(lay)
        parity(got[i], want, f"layer {i}")
        if fp8:
            assert np.array_equal(dl.v_cache.cpu().numpy(), vc)
            assert e4m3_code_distance(dl.k_cache.cpu().numpy(), kc).max() <= 1
        else:
            assert np.array_equal(I.bits(dl.v_cache.cpu()), vc)
            assert bf16_ulp_diff(I.bits(dl.k_cache.cpu()), kc).max() <= 1


def test_serial_equals_the_single_launch_stack_and_is_deterministic():
    L = 20_000
    layers = I.make_stack(L, workload=I.W_STACK_100K + 51)
    a, _ = serial_on_gpu(layers, L - 1)
    b, _ = serial_on_gpu(layers, L - 1)
    assert np.array_equal(a, b)
    dl = [DeviceLayer(l) for l in layers]
    ref = torch.empty((49, 32, 128), dtype=torch.float32, device="cuda")
    flint.flint_attn_stack(dl, L - 1, ref, flint.workspace(49))
    torch.cuda.synchronize()
    # one layer per launch plans each layer over every CTA: same values up to
    # rounding order
    np.testing.assert_allclose(a, ref.cpu().numpy(), rtol=1e-4, atol=1e-5)


def test_serial_100k_sampled_layers():
    L = 100_000
    layers = I.make_stack(L)
    got, dls = serial_on_gpu(layers, L - 1)
    kinds = I.layer_kinds()
    full = [i for i, f in enumerate(kinds) if f]
    for i in (full[0], full[-1], 0, 48):
        want, _, _ = oracle_layer(layers[i])
        parity(got[i], want, f"layer {i}")


def test_both_merge_modes_give_the_same_bits():
    """A full layer at context 100,000, planned alone over every SM (148
    partials), merges on ready flags when it is launched by itself
    (flint_attn_stack of that one layer) and after the grid barrier when it
    is the dependent second launch of the layer-serial path.  The plan, the
    partials and the merge's batch boundaries are the same, so the outputs
    agree bit for bit, and both match the oracle."""
    L = 100_000
    window = I.make_layer(I.W_STACK_100K + 61, 0, L, I.WINDOW, True, ring=True)
    full = I.make_layer(I.W_STACK_100K + 61, 1, L, 0, False, ring=False)
    flags, _ = stack_on_gpu([full], L - 1)
    barrier, _ = serial_on_gpu([window, full], L - 1)
    assert np.array_equal(flags[0], barrier[1])
    want, _, _ = oracle_layer(full)
    parity(flags[0], want, "full layer, ready-flag merge")
