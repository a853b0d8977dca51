"""Pins of the float64 oracle against things other than itself.

Each test ties one oracle function to a library routine (torch's RMSNorm and
SDPA, the rotate-half RoPE of transformers' Llama code, torch's bf16
conversion), to a closed form, to an invariant, or to the numbers printed by
the "Recursive Flint" model JSON.  A dropped term, a wrong sign, a swapped
index or a transposed operand in the oracle fails at least one of them.
"""
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from long_context_decode_flash_b200 import inputs as I

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(7)


def bf16_bits(shape, seed, mean=0.0, std=1.0):
    return I.bits(I.bf16_normal(shape, seed, mean, std))


def f64(bits):
    return torch.from_numpy(bits.astype(np.uint16).view(np.int16).copy()).view(
        torch.bfloat16).to(torch.float64).numpy()


# ---------------------------------------------------------------- bf16 -----

def test_bf16_widening_matches_torch():
    b = rng.integers(0, 1 << 16, size=20000, dtype=np.uint16)
    b = b[(b & 0x7f80) != 0x7f80]  # drop inf / nan patterns
    assert np.array_equal(oracle.bf16_to_f64(b), f64(b))


def test_bf16_rounding_matches_torch_rne_on_float32_values():
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32),
        (rng.standard_normal(2000) * 1e-39).astype(np.float32),   # subnormals
        (rng.standard_normal(2000) * 1e30).astype(np.float32),
    ])
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.f64_to_bf16(x.astype(np.float64)), want)


def test_bf16_rounding_ties_go_to_even():
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: the even neighbour is 1.0.
    # 1 + 3*2^-8 is halfway between 1 + 2^-7 and 1 + 2^-6: the even one is 1 + 2^-6.
    got = oracle.f64_to_bf16(np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8)]))
    assert list(got) == [0x3f80, 0x3f82, 0xbf80]


# ------------------------------------------------------------- RMSNorm -----

def test_rmsnorm_matches_torch_rms_norm():
    x = rng.standard_normal((36, 128)) * 3.0
    w = 1.0 + 0.1 * rng.standard_normal(128)
    want = F.rms_norm(torch.from_numpy(x), (128,), torch.from_numpy(w), eps=1e-6).numpy()
    np.testing.assert_allclose(oracle.rmsnorm(x, w, 1e-6), want, rtol=1e-13, atol=1e-13)


def test_rmsnorm_closed_form_unit_weight():
    # with w = 1, mean(y^2) = ms / (ms + eps) for ms = mean(x^2)
    x = rng.standard_normal((5, 128)) * 1e-3
    eps = 1e-6
    y = oracle.rmsnorm(x, None, eps)
    ms = (x ** 2).mean(axis=1)
    np.testing.assert_allclose((y ** 2).mean(axis=1), ms / (ms + eps), rtol=1e-12)


# ---------------------------------------------------------------- RoPE -----

def _hf_rope(x, pos):
    from transformers import LlamaConfig
    from transformers.models.llama.modeling_llama import (LlamaRotaryEmbedding,
                                                          apply_rotary_pos_emb)
    cfg = LlamaConfig(hidden_size=4096, num_attention_heads=32, head_dim=128,
                      rope_parameters={"rope_type": "default", "rope_theta": 10000.0})
    emb = LlamaRotaryEmbedding(cfg)
    xt = torch.from_numpy(x)[None, :, None, :]            # [1, rows, seq=1, d]
    cos, sin = emb(xt, torch.tensor([[pos]]))
    y, _ = apply_rotary_pos_emb(xt, xt, cos, sin, unsqueeze_dim=1)
    return y[0, :, 0, :].numpy()


@pytest.mark.parametrize("pos", [0, 1, 7, 63])
def test_rope_matches_transformers_rotate_half(pos):
    # transformers forms its angles in float32: use positions where that is exact
    # to ~1e-5 and compare at that tolerance.
    x = rng.standard_normal((6, 128))
    np.testing.assert_allclose(oracle.rope(x, pos), _hf_rope(x, pos), rtol=0, atol=3e-5)


@pytest.mark.parametrize("i,freq", [(0, 1.0), (16, 0.1), (32, 0.01), (48, 0.001)])
def test_rope_closed_form_at_long_context(i, freq):
    # theta^(-2i/128) with theta = 10^4 is 10^(-i/16): exactly these decades.
    pos = 99_999
    e = np.zeros((1, 128))
    e[0, i] = 1.0
    y = oracle.rope(e, pos)
    a = pos * freq
    assert abs(y[0, i] - math.cos(a)) < 1e-9
    assert abs(y[0, i + 64] - math.sin(a)) < 1e-9
    e2 = np.zeros((1, 128))
    e2[0, i + 64] = 1.0
    y2 = oracle.rope(e2, pos)
    assert abs(y2[0, i] + math.sin(a)) < 1e-9
    assert abs(y2[0, i + 64] - math.cos(a)) < 1e-9


def test_rope_invariants():
    q = rng.standard_normal((3, 128))
    k = rng.standard_normal((3, 128))
    np.testing.assert_array_equal(oracle.rope(q, 0), q)
    qr = oracle.rope(q, 123_456)
    np.testing.assert_allclose(np.linalg.norm(qr, axis=1), np.linalg.norm(q, axis=1), rtol=1e-13)
    # the score depends only on the distance m - n
    a = (oracle.rope(q, 100_000) * oracle.rope(k, 99_500)).sum(axis=1)
    b = (oracle.rope(q, 600) * oracle.rope(k, 100)).sum(axis=1)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-9)


# ----------------------------------------------------------- attention -----

def _logical(cache, layout, L, capacity=0, table=None, bs=64):
    """Gather positions 0..L-1 by plain numpy indexing."""
    pos = np.arange(L)
    if layout == oracle.CONTIGUOUS:
        return cache[pos]
    if layout == oracle.RING:
        return cache[pos % capacity]
    flat = cache.reshape((-1,) + cache.shape[2:])
    return flat[np.asarray(table)[pos // bs] * bs + pos % bs]


def sdpa_with_sink(q, K, V, sinks, lo, hi):
    """Library route: torch SDPA in float64 over keys lo..hi-1 plus one extra
    key with zero key and zero value whose logit is set to sink_h through an
    additive mask; q [nq,d], K/V [n,nkv,d] float64."""
    nq, d = q.shape
    nkv = K.shape[1]
    Kt = torch.from_numpy(K[lo:hi]).permute(1, 0, 2)        # [nkv, n, d]
    Vt = torch.from_numpy(V[lo:hi]).permute(1, 0, 2)
    Kt = torch.repeat_interleave(Kt, nq // nkv, dim=0)      # [nq, n, d]
    Vt = torch.repeat_interleave(Vt, nq // nkv, dim=0)
    zero = torch.zeros(nq, 1, d, dtype=torch.float64)
    Kx, Vx = torch.cat([Kt, zero], 1), torch.cat([Vt, zero], 1)
    mask = torch.zeros(nq, 1, hi - lo + 1, dtype=torch.float64)
    mask[:, 0, -1] = torch.from_numpy(np.asarray(sinks, np.float64))
    out = F.scaled_dot_product_attention(torch.from_numpy(q)[:, None, :], Kx, Vx,
                                         attn_mask=mask, scale=1.0 / math.sqrt(d))
    return out[:, 0, :].numpy()


@pytest.mark.parametrize("L,window", [(1, 0), (5, 0), (700, 0), (700, 513), (513, 513),
                                      (514, 513), (3, 513)])
def test_attention_matches_torch_sdpa_contiguous(L, window):
    q = rng.standard_normal((32, 128))
    kc = bf16_bits((L, 4, 128), 11)
    vc = bf16_bits((L, 4, 128), 12)
    sinks = rng.standard_normal(32) * 2
    got = oracle.attn_decode(q, kc, vc, L, sinks, window)
    lo = max(0, L - window) if window else 0
    want = sdpa_with_sink(q, f64(kc), f64(vc), sinks, lo, L)
    np.testing.assert_allclose(got, want, rtol=1e-10, atol=1e-12)


def test_attention_ring_matches_sdpa_over_logical_window():
    L, cap = 2000, 513
    ring = bf16_bits((cap, 4, 128), 21)
    vring = bf16_bits((cap, 4, 128), 22)
    q = rng.standard_normal((32, 128))
    sinks = rng.standard_normal(32)
    got = oracle.attn_decode(q, ring, vring, L, sinks, 513, layout=oracle.RING, capacity=cap)
    K = _logical(ring, oracle.RING, L, cap)
    V = _logical(vring, oracle.RING, L, cap)
    want = sdpa_with_sink(q, f64(K), f64(V), sinks, L - 513, L)
    np.testing.assert_allclose(got, want, rtol=1e-10, atol=1e-12)


def test_attention_paged_permuted_equals_contiguous_exactly():
    L, bs = 1000, 64
    nb = -(-L // bs)
    kc = bf16_bits((nb * bs, 4, 128), 31)
    vc = bf16_bits((nb * bs, 4, 128), 32)
    perm = np.random.default_rng(3).permutation(nb + 5)[:nb].astype(np.int32)
    kp = np.zeros((nb + 5, bs, 4, 128), np.uint16)
    vp = np.zeros_like(kp)
    for j in range(nb):
        kp[perm[j]] = kc[j * bs:(j + 1) * bs]
        vp[perm[j]] = vc[j * bs:(j + 1) * bs]
    q = rng.standard_normal((32, 128))
    sinks = rng.standard_normal(32)
    for window in (0, 513):
        a = oracle.attn_decode(q, kc, vc, L, sinks, window)
        b = oracle.attn_decode(q, kp, vp, L, sinks, window, layout=oracle.PAGED,
                               block_table=perm, block_size=bs)
        np.testing.assert_array_equal(a, b)


def test_sink_to_minus_infinity_is_plain_softmax_attention():
    L = 300
    q = rng.standard_normal((32, 128))
    kc = bf16_bits((L, 4, 128), 41)
    vc = bf16_bits((L, 4, 128), 42)
    got = oracle.attn_decode(q, kc, vc, L, np.full(32, -np.inf))
    K = torch.from_numpy(f64(kc)).permute(1, 0, 2)
    V = torch.from_numpy(f64(vc)).permute(1, 0, 2)
    want = F.scaled_dot_product_attention(torch.from_numpy(q)[None, :, None, :],
                                          K[None], V[None], enable_gqa=True)[0, :, 0].numpy()
    np.testing.assert_allclose(got, want, rtol=1e-10, atol=1e-12)


def test_window_at_least_context_equals_full():
    q = rng.standard_normal((32, 128))
    sinks = rng.standard_normal(32)
    for L in (1, 200, 513):
        kc = bf16_bits((L, 4, 128), 51)
        vc = bf16_bits((L, 4, 128), 52)
        np.testing.assert_array_equal(oracle.attn_decode(q, kc, vc, L, sinks, 513),
                                      oracle.attn_decode(q, kc, vc, L, sinks, 0))


def test_gqa_equals_explicitly_repeated_kv_heads():
    L = 257
    q = rng.standard_normal((32, 128))
    sinks = rng.standard_normal(32)
    kc = bf16_bits((L, 4, 128), 61)
    vc = bf16_bits((L, 4, 128), 62)
    a = oracle.attn_decode(q, kc, vc, L, sinks)
    kr = np.ascontiguousarray(np.repeat(kc, 8, axis=1))   # [L, 32, 128]
    vr = np.ascontiguousarray(np.repeat(vc, 8, axis=1))
    b = oracle.attn_decode(q, kr, vr, L, sinks)
    np.testing.assert_array_equal(a, b)


def test_constant_v_gives_v_times_one_minus_sink_weight():
    L = 400
    q = rng.standard_normal((32, 128))
    sinks = rng.standard_normal(32) + 3.0
    kc = bf16_bits((L, 4, 128), 71)
    c = np.float32(0.71875)                                  # exact in bf16
    vc = np.full((L, 4, 128), np.frombuffer(np.float32(c).tobytes(), np.uint16)[1], np.uint16)
    got = oracle.attn_decode(q, kc, vc, L, sinks)
    K = f64(kc)
    from scipy.special import logsumexp
    for h in range(32):
        s = K[:, h // 8, :] @ q[h] / math.sqrt(128)
        w_sink = math.exp(sinks[h] - logsumexp(np.append(s, sinks[h])))
        np.testing.assert_allclose(got[h], float(c) * (1.0 - w_sink), rtol=1e-12)


# --------------------------------------------------- append and layers -----

def test_append_placement_all_layouts():
    k = bf16_bits((4, 128), 81)
    v = bf16_bits((4, 128), 82)
    # contiguous: row t
    kc = bf16_bits((50, 4, 128), 83)
    vc = bf16_bits((50, 4, 128), 84)
    k0, v0 = kc.copy(), vc.copy()
    oracle.kv_append(kc, vc, oracle.CONTIGUOUS, 37, k, v)
    assert np.array_equal(kc[37], k) and np.array_equal(vc[37], v)
    mask = np.ones(50, bool)
    mask[37] = False
    assert np.array_equal(kc[mask], k0[mask]) and np.array_equal(vc[mask], v0[mask])
    # ring: row t mod 513
    kr = bf16_bits((513, 4, 128), 85)
    vr = bf16_bits((513, 4, 128), 86)
    kr0 = kr.copy()
    oracle.kv_append(kr, vr, oracle.RING, 99_999, k, v, capacity=513)
    assert np.array_equal(kr[99_999 % 513], k) and np.array_equal(vr[99_999 % 513], v)
    mask = np.ones(513, bool)
    mask[99_999 % 513] = False
    assert np.array_equal(kr[mask], kr0[mask])
    # paged: block_table[t // 64] * 64 + t % 64
    table = np.array([5, 2, 7, 0], np.int32)
    kp = bf16_bits((8, 64, 4, 128), 87)
    vp = bf16_bits((8, 64, 4, 128), 88)
    kp0 = kp.copy()
    oracle.kv_append(kp, vp, oracle.PAGED, 150, k, v, block_table=table)
    assert np.array_equal(kp[7, 150 - 128], k) and np.array_equal(vp[7, 22], v)
    kp0[7, 22] = k
    assert np.array_equal(kp, kp0)


def test_qk_norm_rope_chain_matches_library_pipeline():
    # torch rms_norm then transformers' rotate-half RoPE, at a position where
    # the library's float32 angles are accurate
    pos = 9
    q_raw = bf16_bits((32, 128), 91)
    k_raw = bf16_bits((4, 128), 92)
    w_q = bf16_bits((128,), 93, 1.0, 0.1)
    w_k = bf16_bits((128,), 94, 1.0, 0.1)
    q, k, kb = oracle.qk_norm_rope(q_raw, k_raw, w_q, w_k, pos)
    qn = F.rms_norm(torch.from_numpy(f64(q_raw)), (128,), torch.from_numpy(f64(w_q)), 1e-6)
    kn = F.rms_norm(torch.from_numpy(f64(k_raw)), (128,), torch.from_numpy(f64(w_k)), 1e-6)
    np.testing.assert_allclose(q, _hf_rope(qn.numpy(), pos), atol=3e-5)
    np.testing.assert_allclose(k, _hf_rope(kn.numpy(), pos), atol=3e-5)
    want_kb = torch.from_numpy(k.astype(np.float32)).to(torch.bfloat16)
    # bf16 of the f64 value: compare by value within half a bf16 ulp
    np.testing.assert_allclose(f64(kb), k, rtol=2 ** -8)
    assert np.mean(f64(kb) == want_kb.to(torch.float64).numpy()) > 0.99
    # no RoPE, no norm: identity on the bf16 inputs
    q2, k2, _ = oracle.qk_norm_rope(q_raw, k_raw, None, None, pos, apply_rope=False)
    np.testing.assert_array_equal(q2, f64(q_raw))
    np.testing.assert_array_equal(k2, f64(k_raw))


def test_decode_layer_is_append_then_attend_over_library_reference():
    L = 600
    lay = I.make_layer(9, 0, L, 513, True, ring=True)
    kc, vc = I.bits(lay.k_cache).copy(), I.bits(lay.v_cache).copy()
    out = oracle.decode_layer(I.bits(lay.q_raw), I.bits(lay.k_raw), I.bits(lay.v_raw),
                              I.bits(lay.w_q), I.bits(lay.w_k), lay.sinks.numpy(),
                              kc, vc, L, 513, True, layout=oracle.RING, capacity=513)
    # the appended row is the oracle's own k rounded to bf16, and v_raw as is
    q, _, kb = oracle.qk_norm_rope(I.bits(lay.q_raw), I.bits(lay.k_raw), I.bits(lay.w_q),
                                   I.bits(lay.w_k), L - 1)
    slot = (L - 1) % 513
    assert np.array_equal(kc[slot], kb) and np.array_equal(vc[slot], I.bits(lay.v_raw))
    K = _logical(kc, oracle.RING, L, 513)
    V = _logical(vc, oracle.RING, L, 513)
    want = sdpa_with_sink(q, f64(K), f64(V), lay.sinks.numpy().astype(np.float64), L - 513, L)
    np.testing.assert_allclose(out, want, rtol=1e-10, atol=1e-12)


# ---------------------------------------------------------------- sizes ----

def _golden_kv():
    rows = []
    with open(os.path.join(GOLDEN, "kv_cache_gib_per_request.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                c, b, e = line.split()
                rows.append((int(c), float(b), float(e)))
    return rows


def test_kv_bytes_reproduce_the_model_json_table():
    rows = _golden_kv()
    assert len(rows) == 4
    for ctx, gib_bf16, gib_fp8 in rows:
        assert round(oracle.kv_bytes(ctx, elem_bytes=2) / 2 ** 30, 3) == gib_bf16
        assert round(oracle.kv_bytes(ctx, elem_bytes=1) / 2 ** 30, 3) == gib_fp8
    # "28 KiB per token" over the full layers (Model architecture)
    assert oracle.kv_bytes(1000, n_window=0) - oracle.kv_bytes(999, n_window=0) == 28 * 1024


# ------------------------------------------------------ fp8 (e4m3) cache ----
# The "fp8" column of the model JSON's kvCacheGiBPerRequest (one byte per
# value, pinned above) is read as OCP E4M3 with a float32 scale per
# (layer, KV head).  torch's float8_e4m3fn is an independent implementation
# of the same format.

def _torch_e4m3_values():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    return codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_e4m3_decode_matches_torch_for_all_codes():
    got = oracle.e4m3_to_f64(np.arange(256, dtype=np.uint8))
    want = _torch_e4m3_values()
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan) and nan.sum() == 2       # 0x7f, 0xff
    assert np.array_equal(got[~nan], want[~nan])
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9 and got[0x38] == 1.0


def test_e4m3_encode_matches_torch_in_range():
    r = np.random.default_rng(11)
    x = np.concatenate([
        r.normal(0, 30, 20000),                       # normals of both signs
        r.uniform(-2 ** -6, 2 ** -6, 5000),           # subnormal range
        _torch_e4m3_values()[:126] * 1.0,             # every finite code exactly
        # midpoints between neighbouring codes: ties go to the even code
        (_torch_e4m3_values()[1:126] + _torch_e4m3_values()[:125]) / 2,
        np.array([463.9, -463.9, 0.0, -0.0]),
    ])
    x = x[np.abs(x) < 464]
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = oracle.f64_to_e4m3(x)
    assert np.array_equal(got, want)


def test_e4m3_saturates_and_round_trips():
    big = np.array([464.0, 1e6, np.inf, -500.0, -np.inf])
    assert list(oracle.f64_to_e4m3(big)) == [0x7E, 0x7E, 0x7E, 0xFE, 0xFE]
    assert oracle.f64_to_e4m3(np.array([np.nan]))[0] == 0x7F
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    assert np.array_equal(oracle.f64_to_e4m3(oracle.e4m3_to_f64(codes)), codes)


def test_quantize_divides_in_float32_then_rounds():
    r = np.random.default_rng(12)
    x = r.normal(0, 3, 4000)
    for scale in (0.0123, 1.0 / 112, 3.7):
        t = torch.from_numpy(x).to(torch.float32) / torch.tensor(scale, dtype=torch.float32)
        keep = t.abs() < 464
        want = t[keep].to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        got = oracle.quantize_e4m3(x[keep.numpy()], scale)
        assert np.array_equal(got, want)


def _fp8_cache(L, nkv, d, seed):
    r = np.random.default_rng(seed)
    k = r.integers(0, 256, size=(L, nkv, d), dtype=np.uint8)
    v = r.integers(0, 256, size=(L, nkv, d), dtype=np.uint8)
    k[(k & 0x7F) == 0x7F] = 0x01     # no NaN codes
    v[(v & 0x7F) == 0x7F] = 0x02
    return k, v


def test_fp8_attention_equals_bf16_attention_on_the_same_values():
    # With power-of-two scales every dequantized value (4 significant bits)
    # is exact in bf16, so the fp8 path must equal the pinned bf16 path.
    L, nq, nkv, d = 300, 8, 2, 32
    k8, v8 = _fp8_cache(L, nkv, d, 13)
    ks, vs = np.array([2.0 ** -5, 2.0 ** -3], np.float32), np.array([2.0 ** -4, 0.5], np.float32)
    kf = oracle.e4m3_to_f64(k8) * ks[None, :, None]
    vf = oracle.e4m3_to_f64(v8) * vs[None, :, None]
    kb, vb = oracle.f64_to_bf16(kf), oracle.f64_to_bf16(vf)
    assert np.array_equal(oracle.bf16_to_f64(kb), kf) and np.array_equal(oracle.bf16_to_f64(vb), vf)
    q = rng.normal(size=(nq, d))
    sinks = rng.normal(size=nq)
    for window in (0, 64):
        want = oracle.attn_decode(q, kb, vb, L, sinks, window)
        got = oracle.attn_decode_fp8(q, k8, v8, ks, vs, L, sinks, window)
        np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-14)


def test_fp8_attention_with_one_code_everywhere_is_closed_form():
    L, nq, nkv, d = 50, 4, 1, 16
    k8 = np.full((L, nkv, d), 0x30, np.uint8)     # 0.5
    v8 = np.full((L, nkv, d), 0x4B, np.uint8)     # 3.5 * 2^... decoded below
    vs = np.array([0.25], np.float32)
    q = rng.normal(size=(nq, d))
    sinks = np.array([0.3, -1.0, 2.0, -np.inf])
    out = oracle.attn_decode_fp8(q, k8, v8, np.array([1.0], np.float32), vs, L, sinks)
    val = oracle.e4m3_to_f64(np.array([0x4B], np.uint8))[0] * 0.25
    s = q.sum(axis=1) * 0.5 / math.sqrt(d)          # every score of a head is equal
    w = L * np.exp(s) / (L * np.exp(s) + np.exp(sinks))
    np.testing.assert_allclose(out, (w * val)[:, None] * np.ones((1, d)), rtol=1e-12)


@pytest.mark.parametrize("layout", [oracle.CONTIGUOUS, oracle.RING, oracle.PAGED])
def test_fp8_append_places_torch_codes(layout):
    nkv, d, bs = 4, 128, 64
    cap = 513 if layout == oracle.RING else 256
    table = np.array([3, 0, 2, 1], np.int32) if layout == oracle.PAGED else None
    shape = (4 * bs, nkv, d) if layout == oracle.PAGED else (cap, nkv, d)
    kc, vc = np.zeros(shape, np.uint8), np.zeros(shape, np.uint8)
    k = rng.normal(0, 2, size=(nkv, d))
    v = bf16_bits((nkv, d), 99)
    ks = np.array([0.01, 0.02, 0.005, 1.0], np.float32)
    vs = np.array([0.015, 0.25, 0.004, 2.0], np.float32)
    pos = 700 if layout == oracle.RING else 130
    oracle.kv_append_fp8(kc, vc, layout, pos, k, v, ks, vs, capacity=cap, block_table=table)
    if layout == oracle.PAGED:
        row = table[pos // bs] * bs + pos % bs
    else:
        row = pos % 513 if layout == oracle.RING else pos
    tk = torch.from_numpy(k).to(torch.float32) / torch.from_numpy(ks)[:, None]
    tv = torch.from_numpy(f64(v)).to(torch.float32) / torch.from_numpy(vs)[:, None]
    sat = lambda t: t.clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(kc[row], sat(tk)) and np.array_equal(vc[row], sat(tv))
    others = np.ones(shape[0], bool)
    others[row] = False
    assert not kc[others].any() and not vc[others].any()


def test_fp8_decode_layer_is_norm_rope_then_quantized_append_then_attention():
    nq, nkv, d, L, cap = 32, 4, 128, 700, 513
    q_raw, k_raw, v_raw = bf16_bits((nq, d), 201), bf16_bits((nkv, d), 202), bf16_bits((nkv, d), 203)
    w_q, w_k = bf16_bits((d,), 204, 1.0, 0.1), bf16_bits((d,), 205, 1.0, 0.1)
    sinks = rng.normal(size=nq)
    ks = np.array([0.011, 0.009, 0.013, 0.01], np.float32)
    vs = np.array([0.008, 0.012, 0.01, 0.009], np.float32)
    k0, v0 = _fp8_cache(cap, nkv, d, 206)
    kc, vc = k0.copy(), v0.copy()
    got = oracle.decode_layer_fp8(q_raw, k_raw, v_raw, w_q, w_k, sinks, kc, vc, ks, vs, L, 513,
                                  True, layout=oracle.RING, capacity=cap)
    q, k, _ = oracle.qk_norm_rope(q_raw, k_raw, w_q, w_k, L - 1)
    kw, vw = k0.copy(), v0.copy()
    oracle.kv_append_fp8(kw, vw, oracle.RING, L - 1, k, v_raw, ks, vs, capacity=cap)
    assert np.array_equal(kc, kw) and np.array_equal(vc, vw)
    want = oracle.attn_decode_fp8(q, kw, vw, ks, vs, L, sinks, 513, layout=oracle.RING, capacity=cap)
    np.testing.assert_array_equal(got, want)


# ---------------------------------------------------------------- prefill ----

@pytest.mark.parametrize("window,rope", [(0, False), (8, True)])
def test_prefill_rows_match_causal_sdpa_with_a_sink_column(window, rope):
    """Prefill of a T-token prompt: every row of the oracle equals one
    torch SDPA call over the whole prompt with a causal (and sliding-window)
    mask, GQA heads expanded, and the sink as an extra key whose value is
    zero -- the same q, k, v bits on both sides."""
    T, nq, nkv, d = 40, 8, 2, 32
    q_raw, k_raw, v_raw = bf16_bits((T, nq, d), 301), bf16_bits((T, nkv, d), 302), bf16_bits((T, nkv, d), 303)
    w_q, w_k = bf16_bits((d,), 304, 1.0, 0.1), bf16_bits((d,), 305, 1.0, 0.1)
    sinks = rng.normal(size=nq)
    out, qb, kb = oracle.prefill(q_raw, k_raw, v_raw, w_q, w_k, sinks, window, rope, rows=range(T))
    q = torch.from_numpy(f64(qb)).permute(1, 0, 2)                            # [nq, T, d]
    k = torch.from_numpy(f64(kb)).permute(1, 0, 2).repeat_interleave(nq // nkv, 0)
    v = torch.from_numpy(f64(v_raw)).permute(1, 0, 2).repeat_interleave(nq // nkv, 0)
    zero = torch.zeros(nq, 1, d, dtype=torch.float64)
    k = torch.cat([k, zero], dim=1)                                           # sink key at T
    v = torch.cat([v, zero], dim=1)
    t = torch.arange(T)[:, None]
    j = torch.arange(T)[None, :]
    allowed = (j <= t) & ((j > t - window) if window else torch.ones_like(j <= t))
    bias = torch.where(allowed, 0.0, float("-inf")).to(torch.float64)
    bias = bias[None].repeat(nq, 1, 1)
    # the sink column: q . 0 = 0 plus a bias equal to the head's sink logit
    sink_col = torch.from_numpy(sinks).to(torch.float64)[:, None, None].expand(nq, T, 1)
    bias = torch.cat([bias, sink_col * math.sqrt(d)], dim=2) / math.sqrt(d)
    want = F.scaled_dot_product_attention(q, k, v, attn_mask=bias, scale=1.0 / math.sqrt(d))
    np.testing.assert_allclose(out, want.permute(1, 0, 2).numpy(), rtol=1e-10, atol=1e-12)


# ------------------------------------------------------ context parallel ----

def test_partials_over_any_split_merge_to_the_whole_decode():
    """Context-parallel split-KV: the merge of the partials of consecutive
    token ranges equals the decode attention over all of them (the sink
    folded in once), for splits into 1, 2, 3 and 7 uneven ranges."""
    L, nq, nkv, d = 300, 8, 2, 32
    q = rng.normal(size=(nq, d))
    K, V = bf16_bits((L, nkv, d), 411), bf16_bits((L, nkv, d), 412)
    sinks = rng.normal(size=nq)
    want = oracle.attn_decode(q, K, V, L, sinks, 0)
    for cuts in ([], [150], [1, 299], [10, 11, 50, 120, 121, 280]):
        edges = [0] + cuts + [L]
        parts = [oracle.attn_partial(q, K[a:b], V[a:b]) for a, b in zip(edges[:-1], edges[1:])]
        np.testing.assert_allclose(oracle.merge_partials(parts, sinks), want, rtol=1e-12, atol=1e-13)


def test_partial_is_unnormalised_softmax_and_merge_without_sink_is_sdpa():
    """One partial: O / l is plain softmax attention (torch SDPA, no sink),
    m is the row maximum of the log2-scaled scores, and an empty range merges
    as nothing."""
    L, nq, nkv, d = 64, 4, 1, 16
    q = rng.normal(size=(nq, d))
    K, V = bf16_bits((L, nkv, d), 421), bf16_bits((L, nkv, d), 422)
    O, m, lsum = oracle.attn_partial(q, K, V)
    k, v = torch.from_numpy(f64(K)[:, 0, :]), torch.from_numpy(f64(V)[:, 0, :])
    qt = torch.from_numpy(q)
    sdpa = F.scaled_dot_product_attention(qt[None], k[None], v[None]).numpy()[0]
    np.testing.assert_allclose(O / lsum[:, None], sdpa, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(m, (qt @ k.T).numpy().max(axis=1) / math.sqrt(d) * math.log2(math.e), rtol=1e-13)
    empty = oracle.attn_partial(q, K[:0], V[:0])
    assert np.isneginf(empty[1]).all() and (empty[2] == 0).all()
    sinks = np.full(nq, -np.inf)
    np.testing.assert_allclose(oracle.merge_partials([empty, (O, m, lsum)], sinks), sdpa, rtol=1e-12, atol=1e-13)


def test_merge_of_only_empty_partials_with_a_minus_inf_sink_is_zero():
    """No key in any partial and a sink of -inf: no softmax mass anywhere, and
    the merge gives 0 for those heads (not 0/0); heads with a finite sink give
    0 too (the sink carries no value), and a head whose sink is -inf next to
    a non-empty partial is plain softmax attention."""
    nq, d = 4, 16
    q = rng.normal(size=(nq, d))
    K, V = bf16_bits((8, 1, d), 431), bf16_bits((8, 1, d), 432)
    empty = oracle.attn_partial(q, K[:0], V[:0])
    sinks = np.array([-np.inf, -np.inf, 0.5, -3.0])
    out = oracle.merge_partials([empty, empty, empty], sinks)
    assert np.isfinite(out).all() and (out == 0).all()
    full = oracle.attn_partial(q, K, V)
    sinks = np.full(nq, -np.inf)
    want = full[0] / full[2][:, None]
    np.testing.assert_allclose(oracle.merge_partials([empty, full, empty], sinks), want, rtol=1e-12, atol=1e-13)


def test_storage_row_follows_each_layout():
    """Slot of a logical position: contiguous t, ring t mod capacity, paged
    table[t // 64] * 64 + t mod 64 ("Model architecture": window layers keep
    513 tokens; the paged layout is a block table of 64-token blocks)."""
    table = np.array([5, 0, 7, 2], np.int32)
    for t in (0, 1, 63, 64, 100, 255):
        assert oracle.storage_row(oracle.CONTIGUOUS, t) == t
        assert oracle.storage_row(oracle.PAGED, t, block_table=table, block_size=64) == table[t // 64] * 64 + t % 64
    for t in (0, 512, 513, 1025, 100_000):
        assert oracle.storage_row(oracle.RING, t, capacity=513) == t % 513
