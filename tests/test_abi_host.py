"""Host-side checks of libflint.so that need no GPU: the exported symbols,
host arithmetic, argument validation (errors are raised before any CUDA
call), and the split planner's invariants."""
import ctypes
import os
import random
import re

import pytest

from long_context_decode_flash_b200 import flint

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "flint.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(flint_[a-z_0-9]+)\s*\(", src)))


def test_library_exports_every_declared_entry_point():
    lib = flint.load_library()
    names = declared_functions()
    assert len(names) >= 9
    for name in names:
        assert hasattr(lib, name), f"{name} declared in include/flint.h but not exported"
    assert set(names) == set(flint.EXPORTED)


def test_status_strings():
    assert flint.flint_status_string(0) == "ok"
    assert flint.flint_status_string(5) == "device wait timed out"


def test_kv_bytes_matches_the_model_json_table():
    rows = []
    with open(os.path.join(ROOT, "tests", "golden", "kv_cache_gib_per_request.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                c, b, e = line.split()
                rows.append((int(c), float(b), float(e)))
    for ctx, b16, f8 in rows:
        assert round(flint.flint_kv_bytes(ctx) / 2 ** 30, 3) == b16
        assert round(flint.flint_kv_bytes(ctx, elem_bytes=1) / 2 ** 30, 3) == f8
    # the 49-layer read at 100,000 tokens: 14 full layers + 35 windows of 513
    assert flint.flint_kv_bytes(100_000) == 2_903_971_840


def _fake_cache(layout=flint.CONTIGUOUS, capacity=4096):
    c = flint.KVCache()
    c.k, c.v = 0x10000, 0x20000
    c.layout, c.capacity = layout, capacity
    return c


def _decode(cache, seq_lens, window=0, q=0x30000, out=0x40000, ws=0x50000, num_ctas=0):
    lib = flint.load_library()
    arr = (ctypes.c_int32 * len(seq_lens))(*seq_lens)
    return lib.flint_attn_decode(ctypes.c_void_p(q), 0, ctypes.byref(cache), arr, len(seq_lens),
                                 ctypes.c_void_p(0x60000), window, ctypes.c_void_p(out),
                                 ctypes.c_void_p(ws), 1 << 30, num_ctas, None, None)


@pytest.mark.parametrize("kwargs,status", [
    (dict(window=100), flint.FLINT_ERR_UNSUPPORTED),
    (dict(seq_lens=[0]), flint.FLINT_ERR_INVALID_ARG),
    (dict(seq_lens=[5000]), flint.FLINT_ERR_INVALID_ARG),          # beyond capacity 4096
    (dict(seq_lens=[300000]), flint.FLINT_ERR_INVALID_ARG),        # beyond max context
    (dict(seq_lens=[10] * 65), flint.FLINT_ERR_INVALID_ARG),       # batch too large
    (dict(q=0), flint.FLINT_ERR_INVALID_ARG),                      # NULL q
    (dict(out=0x40004), flint.FLINT_ERR_INVALID_ARG),              # misaligned
    (dict(num_ctas=1000), flint.FLINT_ERR_INVALID_ARG),
])
def test_attn_decode_rejects_bad_arguments_on_the_host(kwargs, status):
    seq = kwargs.pop("seq_lens", [100])
    assert _decode(_fake_cache(), seq, **kwargs) == status
    assert flint.flint_last_error() != ""


def test_attn_decode_rejects_bad_caches():
    ring = _fake_cache(flint.RING, 512)
    assert _decode(ring, [100], window=513) == flint.FLINT_ERR_UNSUPPORTED
    ring = _fake_cache(flint.RING, 513)
    assert _decode(ring, [100], window=0) == flint.FLINT_ERR_UNSUPPORTED
    paged = _fake_cache(flint.PAGED, 0)
    assert _decode(paged, [100]) == flint.FLINT_ERR_INVALID_ARG      # no block table
    paged.block_table, paged.block_size, paged.max_blocks_per_req, paged.num_blocks = 0x70000, 32, 4, 8
    assert _decode(paged, [100]) == flint.FLINT_ERR_UNSUPPORTED     # block size 32
    paged.block_size = 64
    assert _decode(paged, [257]) == flint.FLINT_ERR_INVALID_ARG     # 5 blocks > 4
    bad = _fake_cache()
    bad.layout = 7
    assert _decode(bad, [100]) == flint.FLINT_ERR_INVALID_ARG
    bad = _fake_cache()
    bad.req_stride = 12
    assert _decode(bad, [100]) == flint.FLINT_ERR_INVALID_ARG


def test_stack_and_prep_reject_bad_arguments_on_the_host():
    lib = flint.load_library()
    layers = (flint.StackLayer * 1)()
    st = lib.flint_attn_stack(layers, 1, 10, ctypes.c_float(1e-6), ctypes.c_double(1e4),
                              ctypes.c_void_p(0x40000), ctypes.c_void_p(0x50000), 1 << 20, 0, None, None)
    assert st == flint.FLINT_ERR_INVALID_ARG                        # NULL layer pointers
    st = lib.flint_attn_stack(layers, 50, 10, ctypes.c_float(1e-6), ctypes.c_double(1e4),
                              ctypes.c_void_p(0x40000), ctypes.c_void_p(0x50000), 1 << 20, 0, None, None)
    assert st == flint.FLINT_ERR_INVALID_ARG                        # too many layers
    pos = (ctypes.c_int32 * 1)(-1)
    p = ctypes.c_void_p(0x10000)
    st = lib.flint_qk_norm_rope(p, p, p, p, p, pos, 1, ctypes.c_float(1e-6), ctypes.c_double(1e4),
                                1, p, None, None, None, None)
    assert st == flint.FLINT_ERR_INVALID_ARG                        # negative position
    pos = (ctypes.c_int32 * 1)(7)
    c = _fake_cache(capacity=4)
    st = lib.flint_kv_append(p, p, pos, 1, ctypes.byref(c), None, None)
    assert st == flint.FLINT_ERR_INVALID_ARG                        # slot 7 beyond capacity 4


def test_prefill_rejects_bad_arguments_on_the_host():
    lib = flint.load_library()
    p = ctypes.c_void_p(0x10000)
    eps, theta = ctypes.c_float(1e-6), ctypes.c_double(1e4)
    E, U = flint.FLINT_ERR_INVALID_ARG, flint.FLINT_ERR_UNSUPPORTED
    assert lib.flint_prefill_attn(p, p, p, 0, p, 0, p, None, None) == E              # T = 0
    assert lib.flint_prefill_attn(p, p, p, flint.MAX_CONTEXT + 1, p, 0, p, None, None) == E
    assert lib.flint_prefill_attn(p, p, p, 16, p, 100, p, None, None) == U           # window 100
    assert lib.flint_prefill_attn(p, None, p, 16, p, 0, p, None, None) == E           # NULL k
    assert lib.flint_prefill_attn(p, p, ctypes.c_void_p(0x10008), 16, p, 0, p, None, None) == E  # unaligned v
    assert lib.flint_prefill_qk_norm_rope(p, p, p, p, p, 0, eps, theta, 1, p, p, None, None, None, None) == E
    assert lib.flint_prefill_qk_norm_rope(p, p, p, p, p, 16, eps, theta, 2, p, p, None, None, None, None) == E
    assert lib.flint_prefill_qk_norm_rope(p, p, p, p, p, 16, eps, theta, 1, None, None, None, None, None,
                                          None) == E                                   # no output
    assert lib.flint_prefill_qk_norm_rope(p, p, None, p, p, 16, eps, theta, 1, None, None, p, None, None,
                                          None) == E                                   # v_out without v_raw
    c = _fake_cache(capacity=100)
    assert lib.flint_prefill_qk_norm_rope(p, p, p, p, p, 101, eps, theta, 1, p, p, None, ctypes.byref(c),
                                          None, None) == E                             # 101 tokens, 100 slots
    assert "capacity" in lib.flint_last_error().decode()
    assert lib.flint_prefill_qk_norm_rope(p, p, None, p, p, 50, eps, theta, 1, p, p, None, ctypes.byref(c),
                                          None, None) == E                             # cache without v


def test_context_parallel_calls_reject_bad_arguments_on_the_host():
    lib = flint.load_library()
    p = ctypes.c_void_p(0x10000)
    E = flint.FLINT_ERR_INVALID_ARG
    assert lib.flint_merge_partials(p, 0, 1, p, p, None) == E                       # no partials
    assert lib.flint_merge_partials(p, 1025, 1, p, p, None) == E                    # above the maximum
    assert lib.flint_merge_partials(p, 2, 65, p, p, None) == E                      # B too large
    assert lib.flint_merge_partials(ctypes.c_void_p(0x10004), 2, 1, p, p, None) == E  # unaligned
    assert lib.flint_merge_partials(p, 2, 1, None, p, None) == E                    # no sinks
    c = _fake_cache(capacity=100)
    lens = (ctypes.c_int32 * 1)(101)
    st = lib.flint_attn_decode_partial(p, 0, ctypes.byref(c), lens, 1, p, p, 1 << 30, 0, None, None)
    assert st == E and "capacity" in lib.flint_last_error().decode()                 # 101 tokens, 100 slots
    lens = (ctypes.c_int32 * 1)(0)
    assert lib.flint_attn_decode_partial(p, 0, ctypes.byref(c), lens, 1, p, p, 1 << 30, 0, None, None) == E


def test_workspace_bytes_bounds():
    assert flint.flint_attn_workspace_bytes(0, 148) == 0
    assert flint.flint_attn_workspace_bytes(65, 148) == 0
    # room for the largest plan: 768 partials of (32*128 + 2*32) floats
    full = 4096 + 768 * 16640
    assert flint.flint_attn_workspace_bytes(1, 148) == full
    assert flint.flint_attn_workspace_bytes(49, 148) == full


def test_workspace_below_the_static_plan_is_refused_on_the_host():
    # 4 requests of 4,096 tokens (128 tiles each) on 148 CTAs need at least
    # 4096 + (148 + 4) * 16640 bytes; the check comes before any CUDA call
    lib = flint.load_library()
    cache = _fake_cache()
    seq = (ctypes.c_int32 * 4)(*[4096] * 4)
    need = 4096 + (148 + 4) * 16640
    args = (ctypes.c_void_p(0x30000), 0, ctypes.byref(cache), seq, 4, ctypes.c_void_p(0x60000), 0,
            ctypes.c_void_p(0x40000), ctypes.c_void_p(0x50000))
    assert lib.flint_attn_decode(*args, need - 1, 148, None, None) == flint.FLINT_ERR_WORKSPACE
    assert str(need) in flint.flint_last_error()


# ------------------------------------------------------------ planner -----

def check_plan(seg_tiles, G, cost=2):
    items, cb = flint.flint_plan_items(seg_tiles, G, cost)
    assert cb[0] == 0 and cb[-1] == len(items)
    assert all(x <= y for x, y in zip(cb, cb[1:]))
    # every tile of every segment exactly once, items of a segment consecutive
    seen = {}
    last_seg = -1
    for s, t0, t1 in items:
        assert s >= last_seg
        last_seg = s
        assert 0 <= t0 < t1 <= seg_tiles[s]
        seen.setdefault(s, []).append((t0, t1))
    for s, T in enumerate(seg_tiles):
        ranges = seen[s]
        assert ranges[0][0] == 0 and ranges[-1][1] == T
        assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
        for t0, t1 in ranges:
            assert t1 - t0 >= 2 or len(ranges) == 1 or (t0, t1) == ranges[-1]
    # cost balance: no CTA above the mean by more than one item's slack
    loads = [sum(items[i][2] - items[i][1] + cost for i in range(cb[c], cb[c + 1])) for c in range(G)]
    mean = sum(loads) / G
    assert max(loads) <= mean + cost + 3 + 1e-9
    return items, cb, loads


def test_plan_single_full_layer_at_100k():
    # one problem of 100,000 tokens = 3,125 tiles of 32 tokens (all 4 KV heads)
    items, cb, loads = check_plan([3125], 148)
    assert len(items) == 148
    assert min(loads) >= 20


def test_plan_layer_stack_at_100k():
    tiles = [3125 if (i % 7) in (3, 6) else 17 for i in range(49)]
    items, cb, loads = check_plan(tiles, 148)
    assert len(items) <= 148 + 49


def test_plan_random_cases():
    r = random.Random(5)
    for _ in range(200):
        n = r.randint(1, 64)
        tiles = [r.choice([1, 2, 3, 9, r.randint(1, 4096)]) for _ in range(n)]
        G = r.randint(1, 296)
        try:
            check_plan(tiles, G)
        except flint.FlintError:
            # only when the items would not fit one launch
            assert n + G > 512


def test_plan_rejects_bad_arguments():
    with pytest.raises(flint.FlintError):
        flint.flint_plan_items([], 4)
    with pytest.raises(flint.FlintError):
        flint.flint_plan_items([0, 3], 4)


# ------------------------------------------------- planner with a queue -----

def check_split(seg_tiles, G, max_items=768, cost=2):
    items, lists, queue = flint.flint_plan_split(seg_tiles, G, cost, max_items)
    n = len(items)
    assert n <= max_items
    # items sorted by (segment, t0) and tiling every segment exactly
    assert items == sorted(items)
    if sum(seg_tiles) < 64 * G:
        assert queue == []
    for s, T in enumerate(seg_tiles):
        rs = [(t0, t1) for q, t0, t1 in items if q == s]
        assert rs[0][0] == 0 and rs[-1][1] == T
        assert all(a[1] == b[0] and a[0] < a[1] for a, b in zip(rs, rs[1:]))
    # the static lists and the queue name every item exactly once
    named = [i for l in lists for i in l] + queue
    assert sorted(named) == list(range(n))
    # a segment's static items come before its queued chunks, and small
    # segments are never queued
    qset = set(queue)
    for i, (s, t0, t1) in enumerate(items):
        if i in qset:
            assert seg_tiles[s] >= 64
            assert all(items[j][1] < t0 for j in range(n) if items[j][0] == s and j not in qset)
    # the static part is the static planner's plan of the shortened segments
    st = list(seg_tiles)
    for i in queue:
        s, t0, t1 = items[i]
        st[s] -= t1 - t0
    ref_items, ref_cb = flint.flint_plan_items(st, G, cost, max_items)
    static = [[items[i] for i in l] for l in lists]
    assert static == [ref_items[ref_cb[c]:ref_cb[c + 1]] for c in range(G)]
    return items, lists, queue


def test_split_stack_at_100k_queues_the_full_layers_tails():
    tiles = [3125 if (i % 7) in (3, 6) else 17 for i in range(49)]
    items, lists, queue = check_split(tiles, 148)
    queued = sum(items[i][2] - items[i][1] for i in queue)
    assert queued == 14 * (3125 * 200 // 1000)
    # guided sizes: ceil(remaining / 148), at least 8, largest first
    rem, prev = queued, None
    for i in queue:
        size = items[i][2] - items[i][1]
        want = max(8, -(-rem // 148))
        assert size <= want
        rem -= size
    sizes = [items[i][2] - items[i][1] for i in queue]
    assert sizes[0] == -(-queued // 148) and min(sizes) >= 1
    assert len(items) <= 768


def test_split_keeps_short_launches_static():
    # one 100K layer on 148 CTAs is 21 tiles per CTA: no queue
    items, lists, queue = check_split([3125], 148)
    assert queue == [] and len(items) == 148
    # 64 tiles per CTA and more: queued
    assert check_split([64 * 148], 148)[2] != []
    assert check_split([64 * 148 - 1], 148)[2] == []


def test_split_falls_back_to_coarser_queues_then_none():
    tiles = [3125 if (i % 7) in (3, 6) else 17 for i in range(49)]
    full = check_split(tiles, 148)
    small = check_split(tiles, 148, max_items=500)
    assert 0 < len(small[2]) < len(full[2])
    # the no-alloc scratch (251 partials) has no room for a useful queue
    assert check_split(tiles, 148, max_items=251)[2] == []
    static_only = check_split(tiles, 148, max_items=148 + 49)
    assert static_only[2] == []


def test_split_random_cases_and_determinism():
    r = random.Random(11)
    for _ in range(150):
        n = r.randint(1, 64)
        tiles = [r.choice([1, 2, 17, 63, 64, r.randint(1, 8192)]) for _ in range(n)]
        G = r.randint(1, 296)
        try:
            a = check_split(tiles, G)
        except flint.FlintError:
            assert n + G > 768
            continue
        assert a == flint.flint_plan_split(tiles, G)
