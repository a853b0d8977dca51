"""Parity of flint_qk_norm_rope / flint_kv_append against the float64 oracle:
norm/RoPE values, the bf16 k that is appended (within one bf16 ulp of the
oracle's rounding, mismatches counted), and bit-exact cache placement."""
import numpy as np
import pytest
import torch

import oracle
from long_context_decode_flash_b200 import flint
from long_context_decode_flash_b200 import inputs as I

from helpers import bf16_ulp_diff, dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("rope", [False, True])
def test_qk_norm_rope_values(rope):
    B = 6
    pos = [0, 1, 511, 4096, 99_999, 262_143]
    q_raw = I.bf16_normal((B, 32, 128), 501)
    k_raw = I.bf16_normal((B, 4, 128), 502)
    w_q = I.bf16_normal((128,), 503, 1.0, 0.1)
    w_k = I.bf16_normal((128,), 504, 1.0, 0.1)
    q_out = torch.empty((B, 32, 128), dtype=torch.float32, device="cuda")
    k_out = torch.empty((B, 4, 128), dtype=torch.bfloat16, device="cuda")
    flint.flint_qk_norm_rope(dev(q_raw), dev(k_raw), dev(w_q), dev(w_k), pos, apply_rope=rope,
                             q_out=q_out, k_out=k_out)
    torch.cuda.synchronize()
    qg, kg = q_out.cpu().numpy(), I.bits(k_out.cpu())
    worst_ulp, mismatches = 0, 0
    for b in range(B):
        qw, kw, kb = oracle.qk_norm_rope(I.bits(q_raw[b]), I.bits(k_raw[b]), I.bits(w_q),
                                         I.bits(w_k), pos[b], apply_rope=rope)
        np.testing.assert_allclose(qg[b], qw, rtol=0, atol=2e-6 * np.abs(qw).max())
        d = bf16_ulp_diff(kg[b], kb)
        worst_ulp = max(worst_ulp, int(d.max()))
        mismatches += int((d != 0).sum())
    assert worst_ulp <= 1, f"k differs by {worst_ulp} bf16 ulps"
    assert mismatches <= 0.01 * B * 512, f"{mismatches} of {B * 512} k values differ by 1 ulp"


def _caches(layout, B, cap=0, nb=0):
    if layout == flint.PAGED:
        return (I.bf16_normal((nb, 64, 4, 128), 601), I.bf16_normal((nb, 64, 4, 128), 602))
    return I.bf16_normal((B, cap, 4, 128), 603), I.bf16_normal((B, cap, 4, 128), 604)


def _table(B, pos, nb, seed):
    """Block tables of 1563 entries per request drawn from a small pool; the
    blocks that receive the appends are distinct."""
    g = torch.Generator().manual_seed(seed)
    table = torch.randint(0, nb, (B, 1563), generator=g, dtype=torch.int32)
    distinct = torch.randperm(nb, generator=g)[:B].to(torch.int32)
    for b in range(B):
        table[b, pos[b] // 64] = distinct[b]
    return table


@pytest.mark.parametrize("layout", [flint.CONTIGUOUS, flint.RING, flint.PAGED])
def test_kv_append_bit_exact(layout):
    B = 4
    pos = [0, 63, 64, 99_999] if layout != flint.CONTIGUOUS else [0, 63, 64, 1999]
    k = I.bf16_normal((B, 4, 128), 605)
    v = I.bf16_normal((B, 4, 128), 606)
    if layout == flint.PAGED:
        nb = 64
        kc, vc = _caches(layout, B, nb=nb)
        table = _table(B, pos, nb, seed=9)
        cache_args = dict(block_table=dev(table), num_blocks=nb)
    else:
        cap = 513 if layout == flint.RING else 2000
        kc, vc = _caches(layout, B, cap=cap)
        cache_args = dict(capacity=cap)
    kd, vd = dev(kc), dev(vc)
    cache = flint.kv_cache(kd, vd, layout, **cache_args)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    flint.flint_kv_append(dev(k), dev(v), pos, cache, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    want_k, want_v = I.bits(kc).copy(), I.bits(vc).copy()
    for b in range(B):
        if layout == flint.PAGED:
            oracle.kv_append(want_k, want_v, oracle.PAGED, pos[b], I.bits(k[b]), I.bits(v[b]),
                             block_table=table[b].numpy())
        else:
            oracle.kv_append(want_k[b], want_v[b], layout, pos[b], I.bits(k[b]), I.bits(v[b]),
                             capacity=cache_args["capacity"])
    assert np.array_equal(I.bits(kd.cpu()), want_k)
    assert np.array_equal(I.bits(vd.cpu()), want_v)


@pytest.mark.parametrize("layout,rope", [(flint.RING, True), (flint.CONTIGUOUS, False),
                                         (flint.PAGED, True)])
def test_fused_norm_rope_append(layout, rope):
    B = 3
    pos = [5, 777, 99_999] if layout != flint.CONTIGUOUS else [5, 777, 1500]
    q_raw = I.bf16_normal((B, 32, 128), 701)
    k_raw = I.bf16_normal((B, 4, 128), 702)
    v_raw = I.bf16_normal((B, 4, 128), 703)
    w_q = I.bf16_normal((128,), 704, 1.0, 0.1)
    w_k = I.bf16_normal((128,), 705, 1.0, 0.1)
    if layout == flint.PAGED:
        nb = 64
        kc, vc = _caches(layout, B, nb=nb)
        table = _table(B, pos, nb, seed=3)
        cache_args = dict(block_table=dev(table), num_blocks=nb)
    else:
        cap = 513 if layout == flint.RING else 1501
        kc, vc = _caches(layout, B, cap=cap)
        cache_args = dict(capacity=cap)
    kd, vd = dev(kc), dev(vc)
    cache = flint.kv_cache(kd, vd, layout, **cache_args)
    k_out = torch.empty((B, 4, 128), dtype=torch.bfloat16, device="cuda")
    flint.flint_qk_norm_rope(dev(q_raw), dev(k_raw), dev(w_q), dev(w_k), pos, apply_rope=rope,
                             k_out=k_out, v_raw=dev(v_raw), cache=cache)
    torch.cuda.synchronize()
    kg = I.bits(k_out.cpu())
    want_k, want_v = I.bits(kc).copy(), I.bits(vc).copy()
    for b in range(B):
        _, _, kb = oracle.qk_norm_rope(I.bits(q_raw[b]), I.bits(k_raw[b]), I.bits(w_q),
                                       I.bits(w_k), pos[b], apply_rope=rope)
        assert bf16_ulp_diff(kg[b], kb).max() <= 1
        # placement is checked with the GPU's own k bits (rounding is checked above)
        if layout == flint.PAGED:
            oracle.kv_append(want_k, want_v, oracle.PAGED, pos[b], kg[b], I.bits(v_raw[b]),
                             block_table=table[b].numpy())
        else:
            oracle.kv_append(want_k[b], want_v[b], layout, pos[b], kg[b], I.bits(v_raw[b]),
                             capacity=cache_args["capacity"])
    assert np.array_equal(I.bits(kd.cpu()), want_k)
    assert np.array_equal(I.bits(vd.cpu()), want_v)


def test_append_with_bad_block_id_writes_nothing_and_flags():
    nb = 8
    kc, vc = _caches(flint.PAGED, 1, nb=nb)
    table = torch.tensor([[3, 99, 1]], dtype=torch.int32)
    kd, vd = dev(kc), dev(vc)
    cache = flint.kv_cache(kd, vd, flint.PAGED, block_table=dev(table), num_blocks=nb)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    k = I.bf16_normal((1, 4, 128), 801)
    flint.flint_kv_append(dev(k), dev(k), [70], cache, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == flint.FLINT_ERR_INVALID_ARG
    assert np.array_equal(I.bits(kd.cpu()), I.bits(kc))
