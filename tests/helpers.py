"""Shared pieces of the GPU parity tests: device copies of the seeded inputs,
the parity bar, and oracle wrappers for the synthetic layers."""
import numpy as np
import torch

import oracle
from long_context_decode_flash_b200 import flint
from long_context_decode_flash_b200 import inputs as I

# Parity bar for fp32 outputs against the float64 oracle.
MAX_ABS = 2e-3
REL_L2 = 1e-3


def dev(t: torch.Tensor) -> torch.Tensor:
    return t.to("cuda", non_blocking=False).contiguous()


def parity(got, want, what="", per_head=True):
    """Max-abs and relative-L2 bar over the whole output and (per_head) for
    every 128-value row."""
    got = np.asarray(got, np.float64).reshape(-1, want.shape[-1])
    want = np.asarray(want, np.float64).reshape(-1, want.shape[-1])
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = np.abs(got - want)
    rel = np.linalg.norm(got - want) / np.linalg.norm(want)
    rel_head = np.linalg.norm(got - want, axis=1) / np.linalg.norm(want, axis=1)
    assert err.max() <= MAX_ABS, f"{what}: max abs err {err.max():.3e}"
    assert rel <= REL_L2, f"{what}: rel L2 err {rel:.3e}"
    if per_head:
        assert rel_head.max() <= REL_L2, f"{what}: worst head rel L2 {rel_head.max():.3e}"
    return float(err.max()), float(rel)


def bf16_ulp_diff(a_bits: np.ndarray, b_bits: np.ndarray) -> np.ndarray:
    """|a - b| in bf16 ulps for finite bf16 bit patterns of the same sign."""
    def ordered(x):
        x = x.astype(np.int32)
        return np.where(x & 0x8000, 0x8000 - (x & 0x7fff), 0x8000 + (x & 0x7fff))
    return np.abs(ordered(a_bits) - ordered(b_bits))


def u16(t: torch.Tensor) -> np.ndarray:
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


def bf16_values(bits: np.ndarray) -> np.ndarray:
    with np.errstate(invalid="ignore"):  # sentinel slots may hold NaN patterns
        return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def close_bits(got, want, what):
    """bf16 values after norm (+RoPE): float32 on the device, float64 in the
    oracle, each rounded once to bf16.  They differ rarely, and then by one
    ulp -- or, where RoPE's x cos - y sin cancels to near zero, by a few 1e-7
    in absolute terms, which is many ulps of so small a value (the inputs are
    O(1) after the norm); 1e-5 absolute bounds that case."""
    d = bf16_ulp_diff(got, want)
    a, b = bf16_values(got), bf16_values(want)
    with np.errstate(invalid="ignore"):  # sentinel slots may hold inf / NaN patterns (equal bits)
        ok = (d <= 1) | (np.abs(a - b) <= 1e-5)
    assert ok.all(), f"{what}: {int((~ok).sum())} values apart by more than 1 ulp and 1e-5"
    assert (d > 0).mean() <= 0.01, f"{what}: {(d > 0).mean():.4f} of the values differ"


def e4m3_code_distance(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Distance between E4M3 codes in steps of the format (+0 and -0 coincide)."""
    def ordered(x):
        x = x.astype(np.int32)
        return np.where(x & 0x80, -(x & 0x7F), x & 0x7F)
    return np.abs(ordered(a) - ordered(b))


def check_workspace_clean(ws: torch.Tensor):
    """The counter area (the first 4096 bytes) a clean call leaves behind:
    per-problem arrival counters [0, 64) at zero; the grid-barrier word (64)
    with only its generation bit (31) left; queue head (65) and abort word
    (66) at zero; the merge-ticket word (67) with its low 12 bits at zero (its
    upper bits count the launches that ended in merge tickets, the epoch E);
    the spare words up to 128 at zero; the item ready flags [128, 896) each
    zero or the last ticket launch's value (E); the rest zero."""
    w = ws[:4096].view(torch.int32).cpu().numpy().astype(np.int64) & 0xFFFFFFFF
    assert not w[:64].any(), "arrival counters left non-zero"
    assert w[64] & 0x7FFFFFFF == 0, f"grid-barrier word {w[64]:#x}: low bits not back at zero"
    assert not w[65:67].any(), "queue head or abort word left non-zero"
    assert w[67] & 0xFFF == 0, f"ticket word {w[67]:#x}: low bits not back at zero"
    epoch = w[67] >> 12
    assert not w[68:128].any(), "spare counter words left non-zero"
    flags = w[128:896]
    assert np.all((flags == 0) | (flags == epoch)), "an item flag holds another launch's value"
    assert not w[896:].any()


def oracle_layer(layer: I.Layer, nthreads: int = 0):
    """Oracle for one synthetic layer: norm (+RoPE) -> append -> attend.
    Returns (out f64 [32,128], k cache, v cache) after the append: bf16 bits,
    or uint8 codes for an E4M3 layer."""
    if layer.k_scale is not None:
        kc = layer.k_cache.numpy().copy()
        vc = layer.v_cache.numpy().copy()
        out = oracle.decode_layer_fp8(I.bits(layer.q_raw), I.bits(layer.k_raw), I.bits(layer.v_raw),
                                      I.bits(layer.w_q), I.bits(layer.w_k),
                                      layer.sinks.numpy().astype(np.float64), kc, vc,
                                      layer.k_scale, layer.v_scale, layer.L, layer.window,
                                      layer.rope, layout=layer.layout, capacity=layer.capacity,
                                      nthreads=nthreads)
        return out, kc, vc
    kc = I.bits(layer.k_cache).copy()
    vc = I.bits(layer.v_cache).copy()
    out = oracle.decode_layer(I.bits(layer.q_raw), I.bits(layer.k_raw), I.bits(layer.v_raw),
                              I.bits(layer.w_q), I.bits(layer.w_k),
                              layer.sinks.numpy().astype(np.float64), kc, vc, layer.L,
                              layer.window, layer.rope, layout=layer.layout,
                              capacity=layer.capacity, nthreads=nthreads)
    return out, kc, vc


class DeviceLayer:
    """Device copies of a synthetic layer, in the shape flint.stack_layers wants."""

    def __init__(self, layer: I.Layer):
        self.src = layer
        self.q_raw = dev(layer.q_raw)
        self.k_raw = dev(layer.k_raw)
        self.v_raw = dev(layer.v_raw)
        self.w_q = dev(layer.w_q)
        self.w_k = dev(layer.w_k)
        self.sinks = dev(layer.sinks)
        self.k_cache = dev(layer.k_cache)
        self.v_cache = dev(layer.v_cache)
        self.window = layer.window
        self.rope = layer.rope
        self.cache = flint.kv_cache(self.k_cache, self.v_cache, layer.layout,
                                    capacity=layer.capacity, k_scale=layer.k_scale,
                                    v_scale=layer.v_scale)


def stack_on_gpu(layers, pos, num_ctas=0):
    dl = [DeviceLayer(l) for l in layers]
    out = torch.empty((len(dl), 32, 128), dtype=torch.float32, device="cuda")
    ws = flint.workspace(len(dl), num_ctas)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    flint.flint_attn_stack(dl, pos, out, ws, num_ctas=num_ctas, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0, f"device error {int(err.item())}"
    return out.cpu().numpy(), dl
