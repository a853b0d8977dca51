"""Parity of the E4M3 (fp8) KV-cache path against the float64 oracle: the
appended codes, decode over contiguous, ring and paged caches, and the fused
49-layer stack.  The cache holds E4M3 codes of value / scale with one float32
scale per (layer, KV head) for K and for V (the fp8 column of the model
JSON's kvCacheGiBPerRequest; the format is this library's reading)."""
import numpy as np
import pytest
import torch

import oracle
from long_context_decode_flash_b200 import flint
from long_context_decode_flash_b200 import inputs as I

from helpers import DeviceLayer, dev, e4m3_code_distance, oracle_layer, parity, stack_on_gpu

pytestmark = pytest.mark.gpu

W_FP8 = 40  # workload ids of their own for the seeded inputs


def codes(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy()


def run_decode_fp8(q, k, v, seq_lens, sinks, window, ks, vs, layout=flint.CONTIGUOUS, capacity=0,
                   table=None, num_blocks=0, num_ctas=0):
    cache = flint.kv_cache(k, v, layout, capacity=capacity, block_table=table, num_blocks=num_blocks,
                           k_scale=ks, v_scale=vs)
    B = len(seq_lens)
    out = torch.full((B, 32, 128), float("nan"), dtype=torch.float32, device="cuda")
    ws = flint.workspace(B, num_ctas)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    flint.flint_attn_decode(q, cache, seq_lens, sinks, window, out, ws, num_ctas=num_ctas, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return out.cpu().numpy()


@pytest.mark.parametrize("layout", [flint.CONTIGUOUS, flint.RING, flint.PAGED])
def test_fp8_append_of_final_kv_is_bit_exact(layout):
    """flint_kv_append into an E4M3 cache: the codes of float32(x) / scale,
    exactly as the oracle writes them (k and v are bf16, exact in float32)."""
    B, cap = 3, (513 if layout == flint.RING else 640)
    pos = [0, 600, 639] if layout != flint.RING else [0, 700, 1025]
    k = I.bf16_normal((B, 4, 128), 901, 0.0, 3.0)
    v = I.bf16_normal((B, 4, 128), 902, 0.0, 3.0)
    ks, vs = I.fp8_scales(903), I.fp8_scales(904)
    if layout == flint.PAGED:
        nb = 10 * B
        table = torch.randperm(nb, generator=torch.Generator().manual_seed(5)).to(torch.int32).reshape(B, 10)
        shape = (nb, 64, 4, 128)
    else:
        table, nb, shape = None, 0, (B, cap, 4, 128)
    kc0 = torch.randint(0, 256, shape, dtype=torch.uint8, generator=torch.Generator().manual_seed(6))
    vc0 = torch.randint(0, 256, shape, dtype=torch.uint8, generator=torch.Generator().manual_seed(7))
    kd, vd = dev(kc0), dev(vc0)
    cache = flint.kv_cache(kd, vd, layout, capacity=cap if layout != flint.PAGED else 0,
                           block_table=dev(table) if table is not None else None, num_blocks=nb,
                           k_scale=ks, v_scale=vs)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    flint.flint_kv_append(dev(k), dev(v), pos, cache, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    kw, vw = kc0.numpy().copy(), vc0.numpy().copy()
    for b in range(B):
        if layout == flint.PAGED:
            kb, vb, c2, tb = kw, vw, 0, table[b].numpy()
        else:
            kb, vb, c2, tb = kw[b], vw[b], cap, None
        oracle.kv_append_fp8(kb, vb, layout, pos[b], oracle.bf16_to_f64(I.bits(k[b])), I.bits(v[b]),
                             ks, vs, capacity=c2, block_table=tb)
    assert np.array_equal(codes(kd), kw)
    assert np.array_equal(codes(vd), vw)


def test_fp8_norm_rope_append_k_within_one_code():
    """flint_qk_norm_rope into an E4M3 cache: v codes exact; k is the float32
    norm+RoPE on the GPU against float64 in the oracle, so a code may move by
    one step where the value sits at a rounding boundary."""
    B, cap, pos = 4, 300, [5, 130, 200, 299]
    q_raw = I.bf16_normal((B, 32, 128), 911)
    k_raw = I.bf16_normal((B, 4, 128), 912)
    v_raw = I.bf16_normal((B, 4, 128), 913)
    w_q, w_k = I.bf16_normal((128,), 914, 1.0, 0.1), I.bf16_normal((128,), 915, 1.0, 0.1)
    ks, vs = I.fp8_scales(916), I.fp8_scales(917)
    kd = torch.zeros((B, cap, 4, 128), dtype=torch.uint8, device="cuda")
    vd = torch.zeros_like(kd)
    cache = flint.kv_cache(kd, vd, flint.CONTIGUOUS, capacity=cap, k_scale=ks, v_scale=vs)
    q_out = torch.empty((B, 32, 128), dtype=torch.float32, device="cuda")
    flint.flint_qk_norm_rope(dev(q_raw), dev(k_raw), dev(w_q), dev(w_k), pos, apply_rope=True,
                             q_out=q_out, cache=cache, v_raw=dev(v_raw))
    torch.cuda.synchronize()
    kw = np.zeros((B, cap, 4, 128), np.uint8)
    vw = np.zeros_like(kw)
    for b in range(B):
        _, k, _ = oracle.qk_norm_rope(I.bits(q_raw[b]), I.bits(k_raw[b]), I.bits(w_q), I.bits(w_k), pos[b])
        oracle.kv_append_fp8(kw[b], vw[b], oracle.CONTIGUOUS, pos[b], k, I.bits(v_raw[b]), ks, vs,
                             capacity=cap)
    assert np.array_equal(codes(vd), vw)
    d = e4m3_code_distance(codes(kd), kw)
    assert d.max() <= 1 and (d > 0).sum() <= 8


@pytest.mark.parametrize("L", [1, 2, 63, 64, 65, 127, 513, 514, 1000, 5000])
@pytest.mark.parametrize("window", [0, 513])
def test_fp8_decode_contiguous(L, window):
    d = I.make_decode(L, workload=W_FP8, capacity=max(L, 64), fp8=True)
    got = run_decode_fp8(dev(d.q), dev(d.k_cache), dev(d.v_cache), d.seq_lens, dev(d.sinks), window,
                         d.k_scale, d.v_scale, capacity=max(L, 64))
    want = oracle.attn_decode_fp8(I.bits(d.q[0]), codes(d.k_cache[0]), codes(d.v_cache[0]), d.k_scale,
                                  d.v_scale, L, d.sinks.numpy().astype(np.float64), window)
    parity(got[0], want, f"L={L} window={window}")


@pytest.mark.parametrize("window", [0, 513])
def test_fp8_paged_batch(window):
    pb = I.make_paged_batch(seq_lens=[1, 64, 65, 777, 2048, 5000], workload=W_FP8 + 1, fp8=True,
                            spare_blocks=7)
    got = run_decode_fp8(dev(pb.q), dev(pb.k_pool), dev(pb.v_pool), pb.seq_lens, dev(pb.sinks), window,
                         pb.k_scale, pb.v_scale, layout=flint.PAGED, table=dev(pb.block_table),
                         num_blocks=pb.k_pool.shape[0])
    kp, vp = codes(pb.k_pool), codes(pb.v_pool)
    for b, L in enumerate(pb.seq_lens):
        want = oracle.attn_decode_fp8(I.bits(pb.q[b]), kp, vp, pb.k_scale, pb.v_scale, L,
                                      pb.sinks.numpy().astype(np.float64), window, layout=oracle.PAGED,
                                      block_table=pb.block_table[b].numpy())
        parity(got[b], want, f"request {b} L={L} window={window}")


def check_fp8_layer(lay, got, dl, what):
    want, kc, vc = oracle_layer(lay)
    parity(got, want, what)
    k_dev, v_dev = codes(dl.k_cache), codes(dl.v_cache)
    assert np.array_equal(v_dev, vc), f"{what}: v cache differs"
    d = e4m3_code_distance(k_dev, kc)
    assert d.max() <= 1, f"{what}: k codes differ by {d.max()} steps"
    changed = np.argwhere((k_dev != codes(lay.k_cache)).any(axis=(1, 2))).ravel()
    slot = (lay.L - 1) % lay.capacity if lay.layout == flint.RING else lay.L - 1
    assert set(changed.tolist()) <= {slot}, f"{what}: rows {changed} written"


@pytest.mark.parametrize("L", [1, 100, 513, 514, 3000])
def test_fp8_stack_small_context(L):
    layers = I.make_stack(L, workload=W_FP8 + 2, fp8=True)
    got, dls = stack_on_gpu(layers, L - 1)
    for i, (lay, dl) in enumerate(zip(layers, dls)):
        check_fp8_layer(lay, got[i], dl, f"L={L} layer {i}")


def test_fp8_stack_split_invariance_and_determinism():
    L = 9000
    layers = I.make_stack(L, workload=W_FP8 + 3, fp8=True)
    outs = [stack_on_gpu(layers, L - 1, num_ctas=n)[0] for n in (0, 0, 13, 148)]
    assert np.array_equal(outs[0], outs[1])
    for o in outs[2:]:
        np.testing.assert_allclose(o, outs[0], rtol=1e-4, atol=1e-5)


def test_fp8_stack_100k_sampled_layers():
    """The E4M3 stack at context 100,000, launched as the benchmark launches
    it; the oracle checks two full and two window layers (every head) and the
    appended rows of every layer."""
    L = 100_000
    layers = I.make_stack(L, fp8=True)
    got, dls = stack_on_gpu(layers, L - 1)
    kinds = I.layer_kinds()
    full = [i for i, f in enumerate(kinds) if f]
    window = [i for i, f in enumerate(kinds) if not f]
    for i in full[:1] + full[-1:] + window[:1] + window[-1:]:
        check_fp8_layer(layers[i], got[i], dls[i], f"layer {i}")
    assert np.isfinite(got).all()
