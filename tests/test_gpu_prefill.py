"""Parity of the prefill path (the T tokens of one prompt, positions 0..T-1)
against the float64 oracle's prefill: q and k after norm (+RoPE) rounded to
bf16, v converted to fp16 for the PV product, the cache they fill (bf16 and E4M3; contiguous, ring and paged), the
causal attention with sinks on window (513, RoPE) and full (NoPE) layers, and
a decode step that continues from the prefilled cache."""
import numpy as np
import pytest
import torch

import oracle
from long_context_decode_flash_b200 import flint
from long_context_decode_flash_b200 import inputs as I

from helpers import close_bits, dev, e4m3_code_distance, parity, u16

pytestmark = pytest.mark.gpu

W_PF = 50  # workload ids of their own for the seeded inputs


class Dev:
    """Device copies of a PrefillInputs."""

    def __init__(self, p: I.PrefillInputs):
        self.q_raw, self.k_raw, self.v_raw = dev(p.q_raw), dev(p.k_raw), dev(p.v_raw)
        self.w_q, self.w_k, self.sinks = dev(p.w_q), dev(p.w_k), dev(p.sinks)
        self.T, self.window, self.rope = p.q_raw.shape[0], p.window, p.rope


def prep_gpu(d: Dev, cache=None, with_v=False):
    q = torch.empty((d.T, 32, 128), dtype=torch.bfloat16, device="cuda")
    k = torch.empty((d.T, 4, 128), dtype=torch.bfloat16, device="cuda")
    v = torch.empty((d.T, 4, 128), dtype=torch.float16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    flint.flint_prefill_qk_norm_rope(d.q_raw, d.k_raw, d.w_q, d.w_k, apply_rope=d.rope, q_out=q, k_out=k,
                                     v_raw=d.v_raw, v_out=v, cache=cache, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return (q, k, v) if with_v else (q, k)


def f16(v_bf16: torch.Tensor) -> torch.Tensor:
    """The fp16 v operand of the attention-only tests (nearest, as the prep
    kernel converts)."""
    return dev(v_bf16.to(torch.float16))


def attn_gpu(q, k, v, sinks, window):
    T = q.shape[0]
    out = torch.full((T, 32, 128), float("nan"), dtype=torch.float32, device="cuda")
    flint.flint_prefill_attn(q, k, v, sinks, window, out)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def oracle_prefill(p: I.PrefillInputs, rows):
    return oracle.prefill(I.bits(p.q_raw), I.bits(p.k_raw), I.bits(p.v_raw), I.bits(p.w_q), I.bits(p.w_k),
                          p.sinks.numpy().astype(np.float64), p.window, p.rope, rows=rows)


@pytest.mark.parametrize("window", [flint.WINDOW, 0])
def test_prefill_q_and_k_match_the_oracle(window):
    p = I.make_prefill(300, window, workload=W_PF)
    d = Dev(p)
    q, k, v = prep_gpu(d, with_v=True)
    _, qb, kb = oracle_prefill(p, rows=[])
    close_bits(u16(q), qb, "q")
    close_bits(u16(k), kb, "k")
    # v: bf16 -> fp16 to nearest, bit for bit the host conversion
    np.testing.assert_array_equal(v.cpu().view(torch.int16).numpy(), p.v_raw.to(torch.float16).view(torch.int16).numpy())


def test_prefill_v_fp16_at_the_edges_of_the_format():
    """v_out is v_raw converted to fp16 to nearest even, saturating at
    +-65,504 (as documented for flint_prefill_qk_norm_rope): bf16 values
    beyond the fp16 range clamp to the largest finite fp16, values below the
    smallest normal fp16 (6.1e-5) become subnormals or round to zero, signed
    zeros keep their sign; bit for bit a host conversion with the same rule."""
    T = 64
    p = I.make_prefill(T, 0, workload=W_PF + 9)
    edges = torch.tensor([65504.0, 65536.0, -65536.0, 1.0e5, -3.0e38, 3.0e38, 2.0 ** -14, -(2.0 ** -14),
                          2.0 ** -15, 1.5 * 2.0 ** -20, 2.0 ** -24, 2.0 ** -25, 3.0 * 2.0 ** -25,
                          2.0 ** -26, 1e-30, -1e-30, 0.0, -0.0, 6.0e-5, -5.9e-5], dtype=torch.float32)
    v = p.v_raw.clone().reshape(-1)
    idx = torch.arange(edges.numel()) * 97 % v.numel()
    v[idx] = edges.to(torch.bfloat16)
    p.v_raw = v.reshape(T, 4, 128)
    d = Dev(p)
    _, _, v16 = prep_gpu(d, with_v=True)
    want = p.v_raw.float().clamp(-65504.0, 65504.0).to(torch.float16)
    got_bits = v16.cpu().view(torch.int16).numpy()
    want_bits = want.view(torch.int16).numpy()
    np.testing.assert_array_equal(got_bits, want_bits)
    flat = want.reshape(-1)[idx]
    assert (flat[:6].abs() == 65504).all()           # saturated
    assert flat[13].item() == 0.0 and flat[14].item() == 0.0  # below half the smallest subnormal


@pytest.mark.parametrize("T", [1, 2, 15, 16, 17, 64, 65, 200, 700])
@pytest.mark.parametrize("window", [flint.WINDOW, 0])
def test_prefill_attention_every_row(T, window):
    """The attention alone, on the oracle's own q and k bits: every row."""
    p = I.make_prefill(T, window, workload=W_PF + 1)
    want, qb, kb = oracle_prefill(p, rows=range(T))
    q = dev(torch.from_numpy(qb.view(np.int16)).view(torch.bfloat16))
    k = dev(torch.from_numpy(kb.view(np.int16)).view(torch.bfloat16))
    got = attn_gpu(q, k, f16(p.v_raw), dev(p.sinks), window)
    parity(got, want, f"T={T} window={window}")


def check_composed(p, got, q, k, rows, what):
    """Norm (+RoPE) then attention on the device against the oracle's prefill
    from the raw inputs.  q and k are within one bf16 ulp of the oracle's
    (float32 against float64 before the one rounding), and the attention
    meets the bar over the rows t >= 16.  Rows with fewer keys are ill-
    conditioned in q and k: with one of their values one ulp away they move
    by more than the bar (row 5 of the full-layer prompt of
    test_prefill_composed_small moves by 2.3e-3 when q and k are rounded from
    float32 instead of float64, on the CPU alone), so they are held to the
    bar by the attention-only tests, which start from the oracle's own q and
    k bits; here they only have to be finite."""
    want, qb, kb = oracle_prefill(p, rows=rows)
    close_bits(u16(q), qb, "q")
    close_bits(u16(k), kb, "k")
    assert np.isfinite(got[rows]).all()
    keep = [i for i, t in enumerate(rows) if t >= 16]
    parity(got[[rows[i] for i in keep]], want[keep], what, per_head=False)


@pytest.mark.parametrize("window", [flint.WINDOW, 0])
def test_prefill_composed_small(window):
    """Norm (+RoPE) then attention, both on the device, every row of T=1000."""
    T = 1000
    p = I.make_prefill(T, window, workload=W_PF + 2)
    d = Dev(p)
    q, k, v = prep_gpu(d, with_v=True)
    got = attn_gpu(q, k, v, d.sinks, window)
    check_composed(p, got, q, k, list(range(T)), f"window={window}")


def sample_rows(T, seed):
    fixed = [0, 1, 15, 16, 17, 63, 64, 511, 512, 513, 514, 1000, T // 2 - 1, T // 2, T - 17, T - 16, T - 2, T - 1]
    g = np.random.default_rng(seed)
    extra = g.choice(T, size=14, replace=False).tolist()
    return sorted({r for r in fixed + extra if 0 <= r < T})


@pytest.mark.parametrize("window", [flint.WINDOW, 0])
def test_prefill_8192_sampled_rows(window):
    """The 8,192-token prompt: norm (+RoPE) and attention on the device, 32
    sampled rows against the oracle (rows at tile and block edges included)."""
    T = 8192
    p = I.make_prefill(T, window, workload=W_PF + 3)
    d = Dev(p)
    q, k, v = prep_gpu(d, with_v=True)
    got = attn_gpu(q, k, v, d.sinks, window)
    assert np.isfinite(got).all()
    check_composed(p, got, q, k, sample_rows(T, 7), f"T=8192 window={window}")


def test_prefill_attention_ignores_keys_past_the_prompt_and_reruns_identically():
    """Rows depend only on keys <= their own position: the first 100 rows of a
    prompt of 100 tokens equal those of the same prompt continued to 300, bit
    for bit (the same tiles and order of work), and two launches agree."""
    p = I.make_prefill(300, 0, workload=W_PF + 4)
    d = Dev(p)
    q, k, v = prep_gpu(d, with_v=True)
    a = attn_gpu(q, k, v, d.sinks, 0)
    b = attn_gpu(q[:100].contiguous(), k[:100].contiguous(), v[:100].contiguous(), d.sinks, 0)
    c = attn_gpu(q, k, v, d.sinks, 0)
    np.testing.assert_array_equal(a, c)
    np.testing.assert_array_equal(a[:96], b[:96])  # whole 16-row blocks: the same work
    parity(b, a[:100], "prefix")


def caches_for(layout, fp8, T):
    """Device cache tensors filled with a sentinel pattern, the flint_kv_cache
    over them, and the host copies the oracle appends to."""
    g = torch.Generator().manual_seed(11)
    ks, vs = (I.fp8_scales(seed=W_PF + 5), I.fp8_scales(seed=W_PF + 6)) if fp8 else (None, None)
    table = None
    if layout == flint.PAGED:
        nblk = -(-T // 64) + 3
        table = torch.randperm(nblk, generator=g).to(torch.int32)[None, : nblk - 1].contiguous()
        shape, cap, nb = (nblk, 64, 4, 128), 0, nblk
    else:
        cap = flint.WINDOW if layout == flint.RING else T + 40
        shape, nb = (cap, 4, 128), 0
    if fp8:
        kc = torch.randint(0, 256, shape, dtype=torch.uint8, generator=g)
        vc = torch.randint(0, 256, shape, dtype=torch.uint8, generator=g)
    else:
        kc = torch.randint(-32768, 32767, shape, dtype=torch.int16, generator=g).view(torch.bfloat16)
        vc = torch.randint(-32768, 32767, shape, dtype=torch.int16, generator=g).view(torch.bfloat16)
    kd, vd = dev(kc), dev(vc)
    cache = flint.kv_cache(kd, vd, layout, capacity=cap, block_table=dev(table) if table is not None else None,
                           num_blocks=nb, k_scale=ks, v_scale=vs)
    host = (kc.numpy().copy(), vc.numpy().copy()) if fp8 else (I.bits(kc).copy(), I.bits(vc).copy())
    return cache, kd, vd, host, cap, table, ks, vs


@pytest.mark.parametrize("fp8", [False, True])
@pytest.mark.parametrize("layout", [flint.CONTIGUOUS, flint.RING, flint.PAGED])
def test_prefill_fills_the_cache(layout, fp8):
    """Token t lands in slot t of the layout (a ring keeps the last 513 tokens);
    slots no token maps to keep their contents.  v bits (or codes) are exact;
    k is the bf16 k_out bit for bit (bf16) or within one E4M3 step of the
    oracle's code (its float32 value can differ by one bf16 ulp)."""
    T = 1200 if layout == flint.RING else 1000
    window = flint.WINDOW if layout == flint.RING else 0
    p = I.make_prefill(T, window, workload=W_PF + 7)
    d = Dev(p)
    cache, kd, vd, (kh, vh), cap, table, ks, vs = caches_for(layout, fp8, T)
    q, k = prep_gpu(d, cache=cache)
    bt = table.numpy() if table is not None else None
    v_bits = I.bits(p.v_raw)
    for t in range(T):
        qf, kf, kb = oracle.qk_norm_rope(I.bits(p.q_raw[t]), I.bits(p.k_raw[t]), I.bits(p.w_q), I.bits(p.w_k),
                                         t, apply_rope=p.rope)
        if fp8:
            oracle.kv_append_fp8(kh, vh, layout, t, kf, v_bits[t], ks, vs, capacity=cap, block_table=bt)
        else:
            oracle.kv_append(kh, vh, layout, t, kb, v_bits[t], capacity=cap, block_table=bt)
    if fp8:
        kg, vg = kd.cpu().numpy(), vd.cpu().numpy()
        np.testing.assert_array_equal(vg, vh)
        dist = e4m3_code_distance(kg, kh)
        assert dist.max() <= 1 and (dist > 0).mean() <= 0.01
    else:
        kg, vg = u16(kd), u16(vd)
        np.testing.assert_array_equal(vg, vh)
        close_bits(kg, kh, "cached k")
        # and the cached k is the k_out of the same call, bit for bit
        kk = u16(k)
        for t in range(max(0, T - (cap if layout == flint.RING else T)), T):
            row = oracle.storage_row(layout, t, capacity=cap, block_table=bt)
            np.testing.assert_array_equal(kg.reshape(-1, 4, 128)[row], kk[t])


@pytest.mark.parametrize("window", [flint.WINDOW, 0])
def test_decode_continues_from_the_prefilled_cache(window):
    """Prefill T tokens into the cache, then decode token T with the decode
    calls: the result is row T of the oracle's prefill of T + 1 tokens."""
    T = 2000
    p = I.make_prefill(T + 1, window, workload=W_PF + 8)
    head = I.PrefillInputs(p.q_raw[:T], p.k_raw[:T], p.v_raw[:T], p.w_q, p.w_k, p.sinks, window, p.rope)
    d = Dev(head)
    layout = flint.RING if window else flint.CONTIGUOUS
    cap = flint.WINDOW if window else T + 1
    kd = torch.zeros((cap, 4, 128), dtype=torch.bfloat16, device="cuda")
    vd = torch.zeros_like(kd)
    cache = flint.kv_cache(kd, vd, layout, capacity=cap)
    prep_gpu(d, cache=cache)
    q1 = torch.empty((1, 32, 128), dtype=torch.float32, device="cuda")
    flint.flint_qk_norm_rope(dev(p.q_raw[T:]), dev(p.k_raw[T:]), d.w_q, d.w_k, [T], apply_rope=p.rope,
                             q_out=q1, v_raw=dev(p.v_raw[T:]), cache=cache)
    out = torch.full((1, 32, 128), float("nan"), dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    flint.flint_attn_decode(q1, cache, [T + 1], d.sinks, window, out, flint.workspace(1), dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    # (decode keeps q in float32 where prefill rounds it to bf16, so the
    # reference is the oracle's decode of the same step over its own appends)
    kh = np.zeros((cap, 4, 128), np.uint16)
    vh = np.zeros_like(kh)
    for t in range(T):
        _, _, kb = oracle.qk_norm_rope(I.bits(p.q_raw[t]), I.bits(p.k_raw[t]), I.bits(p.w_q), I.bits(p.w_k), t,
                                       apply_rope=p.rope)
        oracle.kv_append(kh, vh, layout, t, kb, I.bits(p.v_raw[t]), capacity=cap)
    dec = oracle.decode_layer(I.bits(p.q_raw[T]), I.bits(p.k_raw[T]), I.bits(p.v_raw[T]), I.bits(p.w_q),
                              I.bits(p.w_k), p.sinks.numpy().astype(np.float64), kh, vh, T + 1, window,
                              p.rope, layout=layout, capacity=cap)
    parity(out.cpu().numpy()[0], dec, "decode after prefill")



def _sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


@pytest.mark.parametrize("which", ["1", "2", "g-1", "g", "g+1", "2g+1"])
def test_prefill_prep_at_the_grid_boundaries(which):
    """The norm/RoPE pass runs a persistent grid of g = 3 x SMs CTAs, each
    over a contiguous share of the tokens: prompts with fewer tokens than
    CTAs, exactly one token per CTA, and one more than that.  q and k are
    within one bf16 ulp of the oracle's, v converts bit for bit, and every
    cached row is the call's own k and raw v."""
    g = 3 * _sms()
    T = {"1": 1, "2": 2, "g-1": g - 1, "g": g, "g+1": g + 1, "2g+1": 2 * g + 1}[which]
    p = I.make_prefill(T, flint.WINDOW, workload=W_PF + 40)
    d = Dev(p)
    kc = torch.zeros((T + 3, 4, 128), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    cache = flint.kv_cache(kc, vc, flint.CONTIGUOUS, capacity=T + 3)
    q, k, v = prep_gpu(d, cache=cache, with_v=True)
    _, qb, kb = oracle_prefill(p, rows=[])
    close_bits(u16(q), qb, "q")
    close_bits(u16(k), kb, "k")
    np.testing.assert_array_equal(u16(v), u16(p.v_raw.to(torch.float16)))
    np.testing.assert_array_equal(u16(kc)[:T], u16(k))
    np.testing.assert_array_equal(u16(vc)[:T], I.bits(p.v_raw))
    assert not u16(kc)[T:].any() and not u16(vc)[T:].any()  # no write past the prompt


@pytest.mark.parametrize("case", ["one unit per CTA", "four CTAs with two units"])
@pytest.mark.parametrize("window", [flint.WINDOW, 0])
def test_prefill_attention_every_row_at_the_unit_deal(case, window):
    """The attention's persistent grid has one CTA per SM, each over units of
    16 query tokens x one KV head: T = 4 x SMs gives one unit per CTA, and 16
    more tokens give four CTAs a second unit.  Every row against the oracle,
    from its own q and k bits."""
    T = 4 * _sms() + (16 if case.startswith("four") else 0)
    p = I.make_prefill(T, window, workload=W_PF + 41)
    want, qb, kb = oracle_prefill(p, rows=range(T))
    q = dev(torch.from_numpy(qb.view(np.int16)).view(torch.bfloat16))
    k = dev(torch.from_numpy(kb.view(np.int16)).view(torch.bfloat16))
    got = attn_gpu(q, k, f16(p.v_raw), dev(p.sinks), window)
    parity(got, want, f"T={T} window={window}")


@pytest.mark.parametrize("window", [flint.WINDOW, 0])
def test_prefill_attention_over_several_rounds_of_units(window):
    """T = 12 x SMs + 16: every CTA walks three or four units, dealt in
    rounds of alternating direction; rows at the edges of 16-token units and
    of 128-key tiles, and a random draw, against the oracle."""
    T = 12 * _sms() + 16
    p = I.make_prefill(T, window, workload=W_PF + 42)
    edges = [0, 1, 15, 16, 17, 127, 128, 129, 511, 512, 513, 514, T // 2, T - 17, T - 16, T - 1]
    rng = np.random.default_rng(7)
    rows = sorted({r for r in edges + rng.choice(T, size=24, replace=False).tolist() if 0 <= r < T})
    want, qb, kb = oracle_prefill(p, rows=rows)
    q = dev(torch.from_numpy(qb.view(np.int16)).view(torch.bfloat16))
    k = dev(torch.from_numpy(kb.view(np.int16)).view(torch.bfloat16))
    got = attn_gpu(q, k, f16(p.v_raw), dev(p.sinks), window)
    parity(got[rows], want, f"T={T} window={window}")


@pytest.mark.parametrize("outputs", ["cache only", "q only", "k only", "q and v", "k, v and cache, no q"])
@pytest.mark.parametrize("rope", [True, False])
def test_prefill_prep_with_a_subset_of_the_outputs(outputs, rope):
    """Each output of the norm/RoPE pass is optional; the kernel stages only
    the rows the call needs (q for q_out, k for k_out or a cache, v for v_out
    or a cache) and expects exactly their bytes.  Every subset must finish
    without a device error and give the same bits as the call with every
    output."""
    T = 700
    window = flint.WINDOW if rope else 0
    p = I.make_prefill(T, window, workload=W_PF + 43)
    d = Dev(p)
    q_ref, k_ref, v_ref = prep_gpu(d, with_v=True)
    want = {"q": u16(q_ref), "k": u16(k_ref), "v": u16(v_ref)}
    use = {"cache only": {"cache"}, "q only": {"q"}, "k only": {"k"}, "q and v": {"q", "v"},
           "k, v and cache, no q": {"k", "v", "cache"}}[outputs]
    q = torch.full((T, 32, 128), float("nan"), dtype=torch.bfloat16, device="cuda") if "q" in use else None
    k = torch.full((T, 4, 128), float("nan"), dtype=torch.bfloat16, device="cuda") if "k" in use else None
    v = torch.full((T, 4, 128), float("nan"), dtype=torch.float16, device="cuda") if "v" in use else None
    cache = None
    if "cache" in use:
        kc = torch.zeros((T, 4, 128), dtype=torch.bfloat16, device="cuda")
        vc = torch.zeros_like(kc)
        cache = flint.kv_cache(kc, vc, flint.CONTIGUOUS, capacity=T)
    needs_v = v is not None or cache is not None
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    flint.flint_prefill_qk_norm_rope(d.q_raw, d.k_raw, d.w_q, d.w_k, apply_rope=d.rope, q_out=q, k_out=k,
                                     v_raw=d.v_raw if needs_v else None, v_out=v, cache=cache, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    if q is not None:
        np.testing.assert_array_equal(u16(q), want["q"])
    if k is not None:
        np.testing.assert_array_equal(u16(k), want["k"])
    if v is not None:
        np.testing.assert_array_equal(u16(v), want["v"])
    if cache is not None:
        np.testing.assert_array_equal(u16(kc), want["k"])
        np.testing.assert_array_equal(u16(vc), I.bits(p.v_raw))
