"""Float64 CPU oracle for Flint decode attention (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports it and shares no code with it.

``flint_oracle.c`` holds the arithmetic; this module builds it with gcc and
marshals numpy arrays through ctypes.  bf16 values travel as uint16 bit
patterns, e4m3 (fp8) cache values as uint8 codes.  Every function is pinned by
tests in ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "flint_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libflint_oracle.so")
_lock = threading.Lock()
_lib = None

# Storage layouts of the oracle's own cache model.
CONTIGUOUS, RING, PAGED = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile flint_oracle.c into libflint_oracle.so (plain -O2, IEEE math)."""
    if force or not os.path.exists(_LIB_PATH) or (
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)):
        tmp = _LIB_PATH + f".{os.getpid()}.tmp"
        subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
                        "-o", tmp, _SRC, "-lm"], check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            I, L, D = ctypes.c_int, ctypes.c_long, ctypes.c_double
            lib.fo_bf16_to_f64_array.argtypes = [P, P, L]
            lib.fo_f64_to_bf16_array.argtypes = [P, P, L]
            lib.fo_rmsnorm_rows.argtypes = [P, I, I, P, D, P]
            lib.fo_rope_rows.argtypes = [P, I, I, L, D]
            lib.fo_qk_norm_rope.argtypes = [P, P, P, P, I, I, I, L, D, D, I, P, P, P]
            lib.fo_storage_row.argtypes = [I, L, I, P, I]
            lib.fo_storage_row.restype = L
            lib.fo_kv_append.argtypes = [P, P, I, I, P, I, I, I, L, P, P]
            lib.fo_attn_decode.argtypes = [P, I, I, I, P, P, I, I, P, I, L, I, P, P, I]
            lib.fo_attn_decode.restype = I
            lib.fo_decode_layer.argtypes = [P, P, P, P, P, P, I, I, I, P, P, I, I, P,
                                            I, L, I, I, D, D, P, I]
            lib.fo_decode_layer.restype = I
            U8, F = ctypes.c_uint8, ctypes.c_float
            lib.fo_e4m3_to_f64.argtypes = [U8]
            lib.fo_e4m3_to_f64.restype = D
            lib.fo_f64_to_e4m3.argtypes = [D]
            lib.fo_f64_to_e4m3.restype = U8
            lib.fo_quantize_e4m3.argtypes = [D, F]
            lib.fo_quantize_e4m3.restype = U8
            lib.fo_kv_append_fp8.argtypes = [P, P, I, I, P, I, I, I, L, P, P, P, P]
            lib.fo_attn_decode_fp8.argtypes = [P, I, I, I, P, P, P, P, I, I, P, I, L, I, P, P, I]
            lib.fo_attn_decode_fp8.restype = I
            lib.fo_decode_layer_fp8.argtypes = [P, P, P, P, P, P, I, I, I, P, P, P, P, I, I, P,
                                                I, L, I, I, D, D, P, I]
            lib.fo_decode_layer_fp8.restype = I
            lib.fo_kv_bytes.argtypes = [L, I, I, I, I, I, I]
            lib.fo_kv_bytes.restype = D
            lib.fo_num_threads.restype = I
            _lib = lib
    return _lib


def _u16(a) -> np.ndarray:
    a = np.asarray(a)
    if a.dtype != np.uint16:
        raise TypeError(f"expected bf16 bit patterns as uint16, got {a.dtype}")
    return np.ascontiguousarray(a)


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return _load().fo_num_threads()


def bf16_to_f64(bits) -> np.ndarray:
    b = _u16(bits)
    out = np.empty(b.shape, np.float64)
    _load().fo_bf16_to_f64_array(_ptr(b), _ptr(out), b.size)
    return out


def f64_to_bf16(x) -> np.ndarray:
    x = _f64(x)
    out = np.empty(x.shape, np.uint16)
    _load().fo_f64_to_bf16_array(_ptr(x), _ptr(out), x.size)
    return out


def rmsnorm(x, w=None, eps: float = 1e-6) -> np.ndarray:
    """x [rows, d] float64, w [d] float64 or None."""
    x = _f64(x)
    rows, d = x.shape
    w = None if w is None else _f64(w)
    y = np.empty_like(x)
    _load().fo_rmsnorm_rows(_ptr(x), rows, d, _ptr(w), eps, _ptr(y))
    return y


def rope(x, pos: int, theta: float = 10000.0) -> np.ndarray:
    """Rotate-half RoPE of rows x [rows, d] at absolute position pos."""
    y = _f64(x).copy()
    rows, d = y.shape
    _load().fo_rope_rows(_ptr(y), rows, d, int(pos), float(theta))
    return y


def qk_norm_rope(q_raw, k_raw, w_q, w_k, pos: int, eps: float = 1e-6,
                 theta: float = 10000.0, apply_rope: bool = True):
    """Returns (q f64 [nq,d], k f64 [nkv,d], k bf16 bits [nkv,d])."""
    q_raw, k_raw = _u16(q_raw), _u16(k_raw)
    w_q = None if w_q is None else _u16(w_q)
    w_k = None if w_k is None else _u16(w_k)
    nq, d = q_raw.shape
    nkv = k_raw.shape[0]
    q = np.empty((nq, d), np.float64)
    k = np.empty((nkv, d), np.float64)
    kb = np.empty((nkv, d), np.uint16)
    _load().fo_qk_norm_rope(_ptr(q_raw), _ptr(k_raw), _ptr(w_q), _ptr(w_k), nq, nkv, d,
                            int(pos), float(eps), float(theta), int(bool(apply_rope)),
                            _ptr(q), _ptr(k), _ptr(kb))
    return q, k, kb


def storage_row(layout: int, pos: int, capacity: int = 0, block_table=None,
                block_size: int = 64) -> int:
    bt = None if block_table is None else np.ascontiguousarray(block_table, np.int32)
    return _load().fo_storage_row(layout, int(pos), int(capacity), _ptr(bt), int(block_size))


def kv_append(k_cache, v_cache, layout: int, pos: int, k, v, capacity: int = 0,
              block_table=None, block_size: int = 64):
    """In place: writes k, v [nkv, d] bf16 bits at pos of uint16 caches whose
    trailing dims are [nkv, d]."""
    for c in (k_cache, v_cache):
        if c.dtype != np.uint16 or not c.flags["C_CONTIGUOUS"]:
            raise TypeError("caches must be C-contiguous uint16 arrays")
    k, v = _u16(k), _u16(v)
    nkv, d = k.shape
    bt = None if block_table is None else np.ascontiguousarray(block_table, np.int32)
    _load().fo_kv_append(_ptr(k_cache), _ptr(v_cache), layout, int(capacity), _ptr(bt),
                         int(block_size), nkv, d, int(pos), _ptr(k), _ptr(v))


def attn_decode(q, k_cache, v_cache, L: int, sinks, window: int = 0,
                layout: int = CONTIGUOUS, capacity: int = 0, block_table=None,
                block_size: int = 64, nthreads: int = 0) -> np.ndarray:
    """One request's decode attention; q [nq, d] float64 (or bf16 bits),
    caches uint16 with trailing dims [nkv, d]; returns float64 [nq, d]."""
    q = bf16_to_f64(q) if np.asarray(q).dtype == np.uint16 else _f64(q)
    nq, d = q.shape
    k_cache, v_cache = _u16(k_cache), _u16(v_cache)
    nkv = k_cache.shape[-2]
    if k_cache.shape[-1] != d:
        raise ValueError("head_dim mismatch")
    sinks = _f64(sinks)
    bt = None if block_table is None else np.ascontiguousarray(block_table, np.int32)
    out = np.empty((nq, d), np.float64)
    rc = _load().fo_attn_decode(_ptr(q), nq, nkv, d, _ptr(k_cache), _ptr(v_cache), layout,
                                int(capacity), _ptr(bt), int(block_size), int(L), int(window),
                                _ptr(sinks), _ptr(out), int(nthreads))
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return out


_LOG2E = 1.4426950408889634


def attn_partial(q, k, v):
    """The unnormalised attention of one query over the keys k / v given
    ([n, nkv, d] bf16 bits; no window, no sink), in log2 units, for a later
    merge across ranks ("Day-0 Support for Flint on vLLM", hnkhoi.com, "Model
    architecture": GQA, query head h reads KV head h / (nq / nkv)):
    s'_j = q_h . k_j / sqrt(d) log2(e), m_h = max_j s'_j,
    l_h = sum_j 2^(s'_j - m_h), O_h = sum_j 2^(s'_j - m_h) v_j.
    q [nq, d] float64 (or bf16 bits).  Returns (O [nq, d], m [nq], l [nq]),
    float64; with no keys m = -inf, l = 0, O = 0."""
    q = bf16_to_f64(q) if np.asarray(q).dtype == np.uint16 else _f64(q)
    nq, d = q.shape
    k, v = bf16_to_f64(k), bf16_to_f64(v)
    n, nkv = k.shape[0], k.shape[1]
    O = np.zeros((nq, d))
    m = np.full(nq, -np.inf)
    lsum = np.zeros(nq)
    if n == 0:
        return O, m, lsum
    for h in range(nq):
        g = h // (nq // nkv)
        s = (k[:, g, :] @ q[h]) / np.sqrt(d) * _LOG2E
        m[h] = s.max()
        w = np.exp2(s - m[h])
        lsum[h] = w.sum()
        O[h] = w @ v[:, g, :]
    return O, m, lsum


def merge_partials(parts, sinks):
    """The log-sum-exp merge of partials (O_r, m_r, l_r) from attn_partial with
    each head's sink logit, which joins the softmax with no value (same page,
    "Learned attention sinks"): M = max(sink log2(e), max_r m_r),
    out = sum_r 2^(m_r - M) O_r / (2^(sink log2(e) - M) + sum_r 2^(m_r - M) l_r).
    A head with no key in any partial and a sink of -inf has no softmax mass
    at all (M = -inf); its output is taken as 0, since nothing carries a value
    (the reading that an empty split adds nothing, never a NaN)."""
    sinks = _f64(sinks) * _LOG2E
    M = sinks.copy()
    for _, m, _ in parts:
        M = np.maximum(M, m)
    empty = np.isneginf(M)
    Mz = np.where(empty, 0.0, M)
    num = 0.0
    den = np.where(np.isneginf(sinks), 0.0, np.exp2(np.where(np.isneginf(sinks), 0.0, sinks) - Mz))
    for O, m, lsum in parts:
        w = np.where(np.isneginf(m), 0.0, np.exp2(np.where(np.isneginf(m), 0.0, m) - Mz))
        num = num + w[:, None] * O
        den = den + w * lsum
    num = num * np.ones((len(M), 1))
    return np.where(empty[:, None], 0.0, num / np.where(empty, 1.0, den)[:, None])


def decode_layer(q_raw, k_raw, v_raw, w_q, w_k, sinks, k_cache, v_cache, L: int,
                 window: int, apply_rope: bool, layout: int = CONTIGUOUS,
                 capacity: int = 0, block_table=None, block_size: int = 64,
                 eps: float = 1e-6, theta: float = 10000.0, nthreads: int = 0):
    """norm (+RoPE) -> append at L-1 -> attend; modifies the caches in place."""
    q_raw, k_raw, v_raw = _u16(q_raw), _u16(k_raw), _u16(v_raw)
    w_q = None if w_q is None else _u16(w_q)
    w_k = None if w_k is None else _u16(w_k)
    for c in (k_cache, v_cache):
        if c.dtype != np.uint16 or not c.flags["C_CONTIGUOUS"]:
            raise TypeError("caches must be C-contiguous uint16 arrays")
    nq, d = q_raw.shape
    nkv = k_raw.shape[0]
    sinks = _f64(sinks)
    bt = None if block_table is None else np.ascontiguousarray(block_table, np.int32)
    out = np.empty((nq, d), np.float64)
    rc = _load().fo_decode_layer(_ptr(q_raw), _ptr(k_raw), _ptr(v_raw), _ptr(w_q), _ptr(w_k),
                                 _ptr(sinks), nq, nkv, d, _ptr(k_cache), _ptr(v_cache), layout,
                                 int(capacity), _ptr(bt), int(block_size), int(L), int(window),
                                 int(bool(apply_rope)), float(eps), float(theta), _ptr(out),
                                 int(nthreads))
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return out


def kv_bytes(ctx: int, n_full: int = 14, n_window: int = 35, window: int = 513,
             nkv: int = 4, d: int = 128, elem_bytes: int = 2) -> float:
    return _load().fo_kv_bytes(int(ctx), n_full, n_window, window, nkv, d, elem_bytes)


# ---- FP8 (e4m3) KV cache --------------------------------------------------

def e4m3_to_f64(codes) -> np.ndarray:
    """Values of e4m3 codes (uint8 array), float64; NaN for S.1111.111."""
    c = np.asarray(codes, np.uint8)
    lib = _load()
    return np.array([lib.fo_e4m3_to_f64(int(x)) for x in c.ravel()], np.float64).reshape(c.shape)


def f64_to_e4m3(x) -> np.ndarray:
    """Nearest e4m3 codes (ties to even, saturating at 448) of float64 values."""
    x = np.asarray(x, np.float64)
    lib = _load()
    return np.array([lib.fo_f64_to_e4m3(float(v)) for v in x.ravel()], np.uint8).reshape(x.shape)


def quantize_e4m3(x, scale: float) -> np.ndarray:
    """Cache codes of x with one scale: float32(x) / float32(scale) in float32,
    then the nearest e4m3 code."""
    x = np.asarray(x, np.float64)
    lib = _load()
    return np.array([lib.fo_quantize_e4m3(float(v), float(scale)) for v in x.ravel()],
                    np.uint8).reshape(x.shape)


def _u8c(c):
    if c.dtype != np.uint8 or not c.flags["C_CONTIGUOUS"]:
        raise TypeError("fp8 caches must be C-contiguous uint8 arrays")
    return c


def _scales(s, nkv):
    s = np.ascontiguousarray(np.asarray(s, np.float32).reshape(-1))
    if s.shape[0] != nkv:
        raise ValueError("one scale per KV head")
    return s


def kv_append_fp8(k_cache, v_cache, layout: int, pos: int, k, v, k_scale, v_scale,
                  capacity: int = 0, block_table=None, block_size: int = 64):
    """In place: quantizes k ([nkv, d] float64) and v ([nkv, d] bf16 bits) into
    uint8 e4m3 caches at pos."""
    _u8c(k_cache), _u8c(v_cache)
    k, v = _f64(k), _u16(v)
    nkv, d = k.shape
    ks, vs = _scales(k_scale, nkv), _scales(v_scale, nkv)
    bt = None if block_table is None else np.ascontiguousarray(block_table, np.int32)
    _load().fo_kv_append_fp8(_ptr(k_cache), _ptr(v_cache), layout, int(capacity), _ptr(bt),
                             int(block_size), nkv, d, int(pos), _ptr(k), _ptr(v), _ptr(ks),
                             _ptr(vs))


def attn_decode_fp8(q, k_cache, v_cache, k_scale, v_scale, L: int, sinks, window: int = 0,
                    layout: int = CONTIGUOUS, capacity: int = 0, block_table=None,
                    block_size: int = 64, nthreads: int = 0) -> np.ndarray:
    """attn_decode over uint8 e4m3 caches with per-KV-head scales."""
    q = bf16_to_f64(q) if np.asarray(q).dtype == np.uint16 else _f64(q)
    nq, d = q.shape
    _u8c(k_cache), _u8c(v_cache)
    nkv = k_cache.shape[-2]
    ks, vs = _scales(k_scale, nkv), _scales(v_scale, nkv)
    sinks = _f64(sinks)
    bt = None if block_table is None else np.ascontiguousarray(block_table, np.int32)
    out = np.empty((nq, d), np.float64)
    rc = _load().fo_attn_decode_fp8(_ptr(q), nq, nkv, d, _ptr(k_cache), _ptr(v_cache), _ptr(ks),
                                    _ptr(vs), layout, int(capacity), _ptr(bt), int(block_size),
                                    int(L), int(window), _ptr(sinks), _ptr(out), int(nthreads))
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return out


def decode_layer_fp8(q_raw, k_raw, v_raw, w_q, w_k, sinks, k_cache, v_cache, k_scale, v_scale,
                     L: int, window: int, apply_rope: bool, layout: int = CONTIGUOUS,
                     capacity: int = 0, block_table=None, block_size: int = 64,
                     eps: float = 1e-6, theta: float = 10000.0, nthreads: int = 0):
    """norm (+RoPE) -> quantized append at L-1 -> attend over e4m3 caches."""
    q_raw, k_raw, v_raw = _u16(q_raw), _u16(k_raw), _u16(v_raw)
    w_q = None if w_q is None else _u16(w_q)
    w_k = None if w_k is None else _u16(w_k)
    _u8c(k_cache), _u8c(v_cache)
    nq, d = q_raw.shape
    nkv = k_raw.shape[0]
    ks, vs = _scales(k_scale, nkv), _scales(v_scale, nkv)
    sinks = _f64(sinks)
    bt = None if block_table is None else np.ascontiguousarray(block_table, np.int32)
    out = np.empty((nq, d), np.float64)
    rc = _load().fo_decode_layer_fp8(_ptr(q_raw), _ptr(k_raw), _ptr(v_raw), _ptr(w_q), _ptr(w_k),
                                     _ptr(sinks), nq, nkv, d, _ptr(k_cache), _ptr(v_cache),
                                     _ptr(ks), _ptr(vs), layout, int(capacity), _ptr(bt),
                                     int(block_size), int(L), int(window), int(bool(apply_rope)),
                                     float(eps), float(theta), _ptr(out), int(nthreads))
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return out


# ---- prefill of a prompt ----------------------------------------------------

def prefill(q_raw, k_raw, v_raw, w_q, w_k, sinks, window: int, apply_rope: bool, rows,
            eps: float = 1e-6, theta: float = 10000.0, nthreads: int = 0):
    """Prefill of a prompt of T tokens at positions 0..T-1 with nothing cached
    before it: per token, norm (+RoPE) of q and k; k rounded to bf16 (the cache
    value) and q rounded to bf16 too (prefill activations are bf16); then query
    row t attends the keys of positions max(0, t - window + 1) .. t (window > 0)
    or 0 .. t, with the head's sink -- the decode attention of position t
    with L = t + 1.  q_raw [T, 32, 128], k_raw / v_raw [T, 4, 128] bf16 bits.
    Returns (out float64 [len(rows), 32, 128] for the requested rows,
    q bf16 bits [T, 32, 128], k bf16 bits [T, 4, 128])."""
    q_raw, k_raw, v_raw = _u16(q_raw), _u16(k_raw), _u16(v_raw)
    T, nq, d = q_raw.shape
    nkv = k_raw.shape[1]
    qb = np.empty((T, nq, d), np.uint16)
    kb = np.empty((T, nkv, d), np.uint16)
    for t in range(T):
        q, _, k16 = qk_norm_rope(q_raw[t], k_raw[t], w_q, w_k, t, eps, theta, apply_rope)
        qb[t] = f64_to_bf16(q)
        kb[t] = k16
    sinks = _f64(sinks)
    out = np.empty((len(rows), nq, d), np.float64)
    for i, t in enumerate(rows):
        out[i] = attn_decode(qb[t], kb, v_raw, int(t) + 1, sinks, window, nthreads=nthreads)
    return out, qb, kb
