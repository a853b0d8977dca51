"""ctypes binding of libflint.so (include/flint.h), argument marshalling only.

Every function here has the name of the C entry point it calls and forwards
device pointers (``tensor.data_ptr()``) and the current CUDA stream.  There is
no fallback: if libflint.so is missing or a call fails, FlintError is raised.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libflint.so")

FLINT_OK = 0
FLINT_ERR_INVALID_ARG = 1
FLINT_ERR_UNSUPPORTED = 2
FLINT_ERR_WORKSPACE = 3
FLINT_ERR_CUDA = 4
FLINT_ERR_TIMEOUT = 5

CONTIGUOUS, RING, PAGED = 0, 1, 2
KV_BF16, KV_FP8_E4M3 = 0, 1
NUM_Q_HEADS, NUM_KV_HEADS, HEAD_DIM = 32, 4, 128
WINDOW, BLOCK_SIZE, MAX_CONTEXT = 513, 64, 262144
MAX_BATCH, MAX_LAYERS = 64, 49

EXPORTED = (
    "flint_status_string", "flint_last_error", "flint_kv_bytes", "flint_qk_norm_rope",
    "flint_kv_append", "flint_attn_workspace_bytes", "flint_attn_decode", "flint_attn_stack",
    "flint_attn_stack_noalloc", "flint_attn_layers_serial", "flint_plan_items", "flint_plan_split",
    "flint_prefill_qk_norm_rope", "flint_prefill_attn", "flint_attn_decode_partial",
    "flint_merge_partials",
)
CP_PARTIAL_FLOATS = 32 * 128 + 2 * 32


class FlintError(RuntimeError):
    def __init__(self, status: int, detail: str):
        super().__init__(f"flint status {status}: {detail}")
        self.status = status


class KVCache(ctypes.Structure):
    """flint_kv_cache.  Build with kv_cache(); it keeps its tensors alive."""
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("layout", ctypes.c_int32),
                ("capacity", ctypes.c_int32), ("req_stride", ctypes.c_int64),
                ("block_table", ctypes.c_void_p), ("max_blocks_per_req", ctypes.c_int32),
                ("block_size", ctypes.c_int32), ("num_blocks", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("k_scale", ctypes.c_float * 4),
                ("v_scale", ctypes.c_float * 4)]


class StackLayer(ctypes.Structure):
    """flint_layer."""
    _fields_ = [("q_raw", ctypes.c_void_p), ("k_raw", ctypes.c_void_p), ("v_raw", ctypes.c_void_p),
                ("w_q", ctypes.c_void_p), ("w_k", ctypes.c_void_p), ("sinks", ctypes.c_void_p),
                ("cache", KVCache), ("window", ctypes.c_int32), ("rope", ctypes.c_int32)]


_lock = threading.Lock()
_lib = None


def open_library(path: str) -> ctypes.CDLL:
    """Load a build of the library from `path` with its signatures declared
    (load_library() does this for the package's libflint.so; tests use it for
    the test builds)."""
    if not os.path.exists(path):
        raise FlintError(FLINT_ERR_CUDA, f"{path} is not built "
                         "(python -m long_context_decode_flash_b200.build)")
    lib = ctypes.CDLL(path)
    P, I32, I64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    lib.flint_status_string.argtypes = [ctypes.c_int]
    lib.flint_status_string.restype = ctypes.c_char_p
    lib.flint_last_error.restype = ctypes.c_char_p
    lib.flint_kv_bytes.argtypes = [I64, I32, I32, I32, I32]
    lib.flint_kv_bytes.restype = ctypes.c_uint64
    lib.flint_qk_norm_rope.argtypes = [P, P, P, P, P, P, I32, ctypes.c_float, ctypes.c_double,
                                       I32, P, P, P, P, P]
    lib.flint_kv_append.argtypes = [P, P, P, I32, P, P, P]
    lib.flint_attn_workspace_bytes.argtypes = [I32, I32]
    lib.flint_attn_workspace_bytes.restype = ctypes.c_size_t
    lib.flint_attn_decode.argtypes = [P, I32, P, P, I32, P, I32, P, P, ctypes.c_size_t,
                                      I32, P, P]
    lib.flint_attn_stack.argtypes = [P, I32, I32, ctypes.c_float, ctypes.c_double, P, P,
                                     ctypes.c_size_t, I32, P, P]
    lib.flint_attn_layers_serial.argtypes = [P, I32, I32, ctypes.c_float, ctypes.c_double, P, P,
                                             ctypes.c_size_t, I32, P, P]
    lib.flint_attn_stack_noalloc.argtypes = [P, I32, I32, ctypes.c_float, ctypes.c_double,
                                             P, I32, P, P]
    lib.flint_prefill_qk_norm_rope.argtypes = [P, P, P, P, P, I32, ctypes.c_float,
                                               ctypes.c_double, I32, P, P, P, P, P, P]
    lib.flint_prefill_attn.argtypes = [P, P, P, I32, P, I32, P, P, P]
    lib.flint_attn_decode_partial.argtypes = [P, I32, P, P, I32, P, P, ctypes.c_size_t, I32, P, P]
    lib.flint_merge_partials.argtypes = [P, I32, I32, P, P, P]
    lib.flint_plan_items.argtypes = [P, I32, I32, I32, P, P, P, P, I32]
    lib.flint_plan_items.restype = I32
    lib.flint_plan_split.argtypes = [P, I32, I32, I32, I32, P, P, P, P, P]
    lib.flint_plan_split.restype = I32
    for name in ("flint_qk_norm_rope", "flint_kv_append", "flint_attn_decode",
                 "flint_attn_stack", "flint_attn_stack_noalloc", "flint_attn_layers_serial",
                 "flint_prefill_qk_norm_rope", "flint_prefill_attn", "flint_attn_decode_partial",
                 "flint_merge_partials"):
        getattr(lib, name).restype = ctypes.c_int
    # test builds only (libflint_hooks.so): leave one pipeline stage unarmed
    for name in ("flint_test_stall_decode", "flint_test_stall_prefill", "flint_test_stall_prefill_prep"):
        if hasattr(lib, name):
            getattr(lib, name).argtypes = [ctypes.c_int, ctypes.c_int]
            getattr(lib, name).restype = ctypes.c_int
    if hasattr(lib, "flint_test_ex2"):  # the prefill softmax's two exponentials, side by side
        lib.flint_test_ex2.argtypes = [P, P, P, I32, P]
        lib.flint_test_ex2.restype = ctypes.c_int
    return lib


def load_library() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            _lib = open_library(LIB_PATH)
    return _lib


def _check(status: int) -> None:
    if status != FLINT_OK:
        lib = load_library()
        raise FlintError(status, lib.flint_last_error().decode())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _i32_host(values: Sequence[int]):
    arr = (ctypes.c_int32 * len(values))(*[int(v) for v in values])
    return arr


def flint_status_string(status: int) -> str:
    return load_library().flint_status_string(int(status)).decode()


def flint_last_error() -> str:
    return load_library().flint_last_error().decode()


def flint_kv_bytes(ctx_len: int, n_full: int = 14, n_window: int = 35, window: int = WINDOW,
                   elem_bytes: int = 2) -> int:
    return int(load_library().flint_kv_bytes(ctx_len, n_full, n_window, window, elem_bytes))


def kv_cache(k: torch.Tensor, v: torch.Tensor, layout: int, capacity: int = 0,
             req_stride: int = 0, block_table: Optional[torch.Tensor] = None,
             num_blocks: int = 0, k_scale: Optional[Sequence[float]] = None,
             v_scale: Optional[Sequence[float]] = None) -> KVCache:
    """A flint_kv_cache over tensors k, v (CONTIGUOUS/RING: [B, cap, 4, 128]
    or [cap, 4, 128]; PAGED: [num_blocks, 64, 4, 128] with an int32 table):
    bf16 tensors, or uint8 tensors of E4M3 codes with k_scale and v_scale
    (4 floats each, one per KV head)."""
    c = KVCache()
    if k.dtype == torch.uint8:
        if k_scale is None or v_scale is None or len(k_scale) != 4 or len(v_scale) != 4:
            raise FlintError(FLINT_ERR_INVALID_ARG, "an E4M3 cache needs 4 k_scale and 4 v_scale values")
        c.dtype = KV_FP8_E4M3
        c.k_scale[:] = [float(x) for x in k_scale]
        c.v_scale[:] = [float(x) for x in v_scale]
    elif k.dtype != torch.bfloat16:
        raise FlintError(FLINT_ERR_INVALID_ARG, f"cache tensors must be bf16 or uint8, not {k.dtype}")
    c.k, c.v = k.data_ptr(), v.data_ptr()
    c.layout = int(layout)
    c.capacity = int(capacity)
    c.req_stride = int(req_stride)
    c.block_table = block_table.data_ptr() if block_table is not None else None
    c.max_blocks_per_req = int(block_table.shape[-1]) if block_table is not None else 0
    c.block_size = BLOCK_SIZE if layout == PAGED else 0
    c.num_blocks = int(num_blocks)
    c._keep = (k, v, block_table)  # keep the tensors alive with the struct
    return c


def flint_attn_workspace_bytes(n_problems: int, num_ctas: int = 0) -> int:
    return int(load_library().flint_attn_workspace_bytes(n_problems, num_ctas))


def workspace(n_problems: int, num_ctas: int = 0, device=None) -> torch.Tensor:
    """A zero-filled workspace of the required size (the library keeps it zeroed)."""
    n = flint_attn_workspace_bytes(n_problems, num_ctas)
    if n == 0:
        raise FlintError(FLINT_ERR_INVALID_ARG, "invalid workspace request")
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def flint_qk_norm_rope(q_raw, k_raw, w_q, w_k, pos: Sequence[int], eps: float = 1e-6,
                       theta: float = 10000.0, apply_rope: bool = True, q_out=None, k_out=None,
                       v_raw=None, cache: Optional[KVCache] = None, dev_err=None, stream=None):
    B = len(pos)
    lib = load_library()
    _check(lib.flint_qk_norm_rope(_ptr(q_raw), _ptr(k_raw), _ptr(v_raw), _ptr(w_q), _ptr(w_k),
                                  _i32_host(pos), B, eps, theta, int(bool(apply_rope)),
                                  _ptr(q_out), _ptr(k_out),
                                  ctypes.byref(cache) if cache is not None else None,
                                  _ptr(dev_err), _stream(stream)))
    return q_out, k_out


def flint_kv_append(k, v, pos: Sequence[int], cache: KVCache, dev_err=None, stream=None) -> None:
    lib = load_library()
    _check(lib.flint_kv_append(_ptr(k), _ptr(v), _i32_host(pos), len(pos), ctypes.byref(cache),
                               _ptr(dev_err), _stream(stream)))


def flint_prefill_qk_norm_rope(q_raw, k_raw, w_q, w_k, eps: float = 1e-6, theta: float = 10000.0,
                               apply_rope: bool = True, q_out=None, k_out=None, v_raw=None, v_out=None,
                               cache: Optional[KVCache] = None, dev_err=None, stream=None):
    """Norm (+RoPE) of the T tokens of one prompt at positions 0..T-1: q and k
    out in bf16, v out in fp16 (the attention's v operand), optional cache
    write (request 0 of `cache`)."""
    T = int(q_raw.shape[0])
    lib = load_library()
    _check(lib.flint_prefill_qk_norm_rope(_ptr(q_raw), _ptr(k_raw), _ptr(v_raw), _ptr(w_q), _ptr(w_k),
                                          T, eps, theta, int(bool(apply_rope)), _ptr(q_out),
                                          _ptr(k_out), _ptr(v_out),
                                          ctypes.byref(cache) if cache is not None else None,
                                          _ptr(dev_err), _stream(stream)))
    return q_out, k_out, v_out


def flint_prefill_attn(q, k, v, sinks, window: int, out, dev_err=None, stream=None):
    """Causal attention (with sinks) of a T-token prompt over itself:
    q bf16 [T, 32, 128], k bf16 [T, 4, 128], v fp16 [T, 4, 128],
    out fp32 [T, 32, 128]."""
    lib = load_library()
    _check(lib.flint_prefill_attn(_ptr(q), _ptr(k), _ptr(v), int(q.shape[0]), _ptr(sinks), int(window),
                                  _ptr(out), _ptr(dev_err), _stream(stream)))
    return out


def flint_attn_decode(q, cache: KVCache, seq_lens: Sequence[int], sinks, window: int, out,
                      ws: torch.Tensor, num_ctas: int = 0, dev_err=None, stream=None):
    if q.dtype not in (torch.bfloat16, torch.float32):
        raise FlintError(FLINT_ERR_INVALID_ARG, "q must be bf16 or fp32")
    lib = load_library()
    _check(lib.flint_attn_decode(_ptr(q), int(q.dtype == torch.float32), ctypes.byref(cache),
                                 _i32_host(seq_lens), len(seq_lens), _ptr(sinks), int(window),
                                 _ptr(out), _ptr(ws), ws.numel() * ws.element_size(), int(num_ctas),
                                 _ptr(dev_err), _stream(stream)))
    return out


def flint_attn_decode_partial(q, cache: KVCache, seq_lens: Sequence[int], partials, ws: torch.Tensor,
                              num_ctas: int = 0, dev_err=None, stream=None):
    """This rank's unnormalised attention over tokens [0, seq_lens[b]) of its
    cache: partials fp32 [B, CP_PARTIAL_FLOATS] (O [32,128], m [32], l [32])."""
    if q.dtype not in (torch.bfloat16, torch.float32):
        raise FlintError(FLINT_ERR_INVALID_ARG, "q must be bf16 or fp32")
    lib = load_library()
    _check(lib.flint_attn_decode_partial(_ptr(q), int(q.dtype == torch.float32), ctypes.byref(cache),
                                         _i32_host(seq_lens), len(seq_lens), _ptr(partials), _ptr(ws),
                                         ws.numel() * ws.element_size(), int(num_ctas), _ptr(dev_err),
                                         _stream(stream)))
    return partials


def flint_merge_partials(partials, sinks, out, stream=None):
    """Merge partials fp32 [n_parts, B, CP_PARTIAL_FLOATS] with the sinks into
    out fp32 [B, 32, 128]."""
    n, B = int(partials.shape[0]), int(partials.shape[1])
    lib = load_library()
    _check(lib.flint_merge_partials(_ptr(partials), n, B, _ptr(sinks), _ptr(out), _stream(stream)))
    return out


def stack_layers(layers) -> ctypes.Array:
    """A flint_layer array from objects with q_raw, k_raw, v_raw, w_q, w_k, sinks
    (device tensors), cache (KVCache), window and rope."""
    arr = (StackLayer * len(layers))()
    keep = []
    for i, ly in enumerate(layers):
        s = arr[i]
        s.q_raw, s.k_raw, s.v_raw = ly.q_raw.data_ptr(), ly.k_raw.data_ptr(), ly.v_raw.data_ptr()
        s.w_q, s.w_k, s.sinks = ly.w_q.data_ptr(), ly.w_k.data_ptr(), ly.sinks.data_ptr()
        s.cache = ly.cache
        s.window = int(ly.window)
        s.rope = int(bool(ly.rope))
        keep.append(ly)
    arr._keep = keep
    return arr


def flint_attn_stack(layers, pos: int, out, ws: torch.Tensor, eps: float = 1e-6,
                     theta: float = 10000.0, num_ctas: int = 0, dev_err=None, stream=None):
    """layers: a ctypes array from stack_layers() (or a list, converted here)."""
    arr = layers if isinstance(layers, ctypes.Array) else stack_layers(layers)
    lib = load_library()
    _check(lib.flint_attn_stack(arr, len(arr), int(pos), eps, theta, _ptr(out), _ptr(ws),
                                ws.numel() * ws.element_size(), int(num_ctas), _ptr(dev_err),
                                _stream(stream)))
    return out


def flint_attn_layers_serial(layers, pos: int, out, ws: torch.Tensor, eps: float = 1e-6,
                             theta: float = 10000.0, num_ctas: int = 0, dev_err=None, stream=None):
    """flint_attn_stack as one dependent launch per layer (programmatic
    dependent launch); layers: a ctypes array from stack_layers() or a list."""
    arr = layers if isinstance(layers, ctypes.Array) else stack_layers(layers)
    lib = load_library()
    _check(lib.flint_attn_layers_serial(arr, len(arr), int(pos), eps, theta, _ptr(out), _ptr(ws),
                                        ws.numel() * ws.element_size(), int(num_ctas), _ptr(dev_err),
                                        _stream(stream)))
    return out


def flint_attn_stack_noalloc(layers, pos: int, out, eps: float = 1e-6, theta: float = 10000.0,
                             num_ctas: int = 0, dev_err=None, stream=None):
    """flint_attn_stack on the library's own fixed device scratch (no workspace)."""
    arr = layers if isinstance(layers, ctypes.Array) else stack_layers(layers)
    lib = load_library()
    _check(lib.flint_attn_stack_noalloc(arr, len(arr), int(pos), eps, theta, _ptr(out),
                                        int(num_ctas), _ptr(dev_err), _stream(stream)))
    return out


def flint_plan_items(seg_tiles: Sequence[int], num_ctas: int, item_cost: int = 2,
                     max_items: int = 512):
    """Returns (items [(seg, t0, t1)], cta_begin list) from the C planner."""
    n = len(seg_tiles)
    st = _i32_host(seg_tiles)
    seg = (ctypes.c_int32 * max_items)()
    t0 = (ctypes.c_int32 * max_items)()
    t1 = (ctypes.c_int32 * max_items)()
    cb = (ctypes.c_int32 * (num_ctas + 1))()
    k = load_library().flint_plan_items(st, n, num_ctas, item_cost, seg, t0, t1, cb, max_items)
    if k < 0:
        raise FlintError(FLINT_ERR_INVALID_ARG, "planner rejected the arguments")
    return [(seg[i], t0[i], t1[i]) for i in range(k)], list(cb)


def flint_plan_split(seg_tiles: Sequence[int], num_ctas: int, item_cost: int = 2,
                     max_items: int = 768):
    """Returns (items [(seg, t0, t1)] sorted by segment, static lists [[item
    index, ...] per CTA], queue [item index, ...]) from the C planner."""
    n = len(seg_tiles)
    st = _i32_host(seg_tiles)
    seg = (ctypes.c_int32 * max_items)()
    t0 = (ctypes.c_int32 * max_items)()
    t1 = (ctypes.c_int32 * max_items)()
    order = (ctypes.c_int32 * max_items)()
    cb = (ctypes.c_int32 * (num_ctas + 1))()
    k = load_library().flint_plan_split(st, n, num_ctas, item_cost, max_items, seg, t0, t1, order, cb)
    if k < 0:
        raise FlintError(FLINT_ERR_INVALID_ARG, "planner rejected the arguments")
    items = [(seg[i], t0[i], t1[i]) for i in range(k)]
    lists = [[order[j] for j in range(cb[c], cb[c + 1])] for c in range(num_ctas)]
    queue = [order[j] for j in range(cb[num_ctas], k)]
    return items, lists, queue
