"""Seeded synthetic inputs for Flint decode attention.

This module only draws random numbers and arranges them into the shapes of the
workloads; it holds none of the attention arithmetic.  The CUDA path and the
CPU oracle both consume exactly the tensors produced here (the oracle through
their uint16 bit patterns), so both sides see the same bf16 values.

Recipe (the pages ship no data, prompts or weights, so synthetic tensors
stand in for them):
  * q, k, v, K/V caches: bf16 ~ N(0, 1)  (float32 normal draw, then
    round-to-nearest-even to bf16 by torch's conversion)
  * sink logits: float32 ~ N(0, 1), one per query head
  * Q/K RMSNorm weights: bf16 ~ 1 + N(0, 0.1), one [128] vector each for q
    and k per layer
  * paged batches: context lengths log-uniform in [4096, 131072], 64-token
    blocks, block ids a random permutation of the pool
Every tensor has its own seed: BASE_SEED + 1000 * workload + 16 * layer +
tensor id, drawn with torch's CPU generator (independent of thread count).
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional

import numpy as np
import torch

BASE_SEED = 20261202

NUM_Q_HEADS = 32
NUM_KV_HEADS = 4
HEAD_DIM = 128
WINDOW = 513
BLOCK_SIZE = 64
N_LAYERS = 49

# workload ids used in seeds
W_FULL_SMALL, W_SWA_100K, W_FULL_100K, W_STACK_100K, W_PAGED_BATCH, W_PREFILL = 0, 1, 2, 3, 4, 5

# tensor ids inside a layer
_T_Q, _T_K, _T_V, _T_WQ, _T_WK, _T_SINK, _T_KC, _T_VC = range(8)

CONTIGUOUS, RING, PAGED = 0, 1, 2


def seed_for(workload: int, layer: int, tensor: int) -> int:
    return BASE_SEED + 1000 * workload + 16 * layer + tensor


def _gen(seed: int) -> torch.Generator:
    return torch.Generator().manual_seed(int(seed))


def bf16_normal(shape, seed: int, mean: float = 0.0, std: float = 1.0) -> torch.Tensor:
    """bf16 CPU tensor ~ N(mean, std^2) (float32 draw rounded to bf16)."""
    x = torch.randn(tuple(shape), generator=_gen(seed), dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    if mean != 0.0:
        x.add_(mean)
    return x.to(torch.bfloat16)


def f32_normal(shape, seed: int) -> torch.Tensor:
    return torch.randn(tuple(shape), generator=_gen(seed), dtype=torch.float32)


def bits(t: torch.Tensor) -> np.ndarray:
    """uint16 bit patterns of a bf16 CPU tensor (shares memory)."""
    assert t.dtype == torch.bfloat16 and t.device.type == "cpu"
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


@dataclasses.dataclass
class Layer:
    """One attention layer of one decode step for one request."""
    window: int                      # 0 = full context, else 513
    rope: bool
    L: int                           # tokens valid after the append (new token at L-1)
    q_raw: torch.Tensor              # bf16 [32,128]
    k_raw: torch.Tensor              # bf16 [4,128]
    v_raw: torch.Tensor              # bf16 [4,128]
    w_q: torch.Tensor                # bf16 [128]
    w_k: torch.Tensor                # bf16 [128]
    sinks: torch.Tensor              # f32 [32]
    k_cache: torch.Tensor            # bf16 [capacity,4,128], or uint8 E4M3 codes
    v_cache: torch.Tensor
    layout: int                      # CONTIGUOUS or RING
    capacity: int
    k_scale: Optional[List[float]] = None   # E4M3 cache: per KV head
    v_scale: Optional[List[float]] = None


# E4M3 (fp8) caches hold the same N(0, 1) history as the bf16 ones, divided by
# a per-KV-head scale and cast to torch.float8_e4m3fn (torch's conversion,
# nearest even, after a clamp to the largest code): the scales put |x| = 6 near
# the top code 448.  Scales are drawn per (workload, layer, K/V).
_T_KS, _T_VS = 8, 9


def fp8_scales(seed: int) -> List[float]:
    u = torch.rand(NUM_KV_HEADS, generator=_gen(seed), dtype=torch.float64)
    return [float(6.0 / 448.0 * (0.9 + 0.2 * x)) for x in u]


def to_e4m3_codes(x: torch.Tensor, scales: List[float]) -> torch.Tensor:
    """uint8 E4M3 codes of x [..., 4, 128] / scales[kv head], via torch's cast."""
    s = torch.tensor(scales, dtype=torch.float32).reshape(NUM_KV_HEADS, 1)
    y = (x.to(torch.float32) / s).clamp(-448.0, 448.0)
    return y.to(torch.float8_e4m3fn).view(torch.uint8)


def make_layer(workload: int, layer: int, L: int, window: int, rope: bool,
               ring: Optional[bool] = None, capacity: Optional[int] = None,
               fp8: bool = False) -> Layer:
    """A layer whose cache holds random history for positions < L-1.

    Window layers use a 513-slot ring unless ring=False; full layers use a
    contiguous cache with `capacity` (default L) slots."""
    if ring is None:
        ring = window > 0
    if ring:
        layout, cap = RING, WINDOW
    else:
        layout, cap = CONTIGUOUS, (capacity if capacity is not None else L)
    s = lambda t: seed_for(workload, layer, t)  # noqa: E731
    k_cache = bf16_normal((cap, NUM_KV_HEADS, HEAD_DIM), s(_T_KC))
    v_cache = bf16_normal((cap, NUM_KV_HEADS, HEAD_DIM), s(_T_VC))
    k_scale = v_scale = None
    if fp8:
        k_scale, v_scale = fp8_scales(s(_T_KS)), fp8_scales(s(_T_VS))
        k_cache, v_cache = to_e4m3_codes(k_cache, k_scale), to_e4m3_codes(v_cache, v_scale)
    return Layer(
        window=window, rope=rope, L=L,
        q_raw=bf16_normal((NUM_Q_HEADS, HEAD_DIM), s(_T_Q)),
        k_raw=bf16_normal((NUM_KV_HEADS, HEAD_DIM), s(_T_K)),
        v_raw=bf16_normal((NUM_KV_HEADS, HEAD_DIM), s(_T_V)),
        w_q=bf16_normal((HEAD_DIM,), s(_T_WQ), 1.0, 0.1),
        w_k=bf16_normal((HEAD_DIM,), s(_T_WK), 1.0, 0.1),
        sinks=f32_normal((NUM_Q_HEADS,), s(_T_SINK)),
        k_cache=k_cache, v_cache=v_cache,
        layout=layout, capacity=cap, k_scale=k_scale, v_scale=v_scale)


def layer_kinds(n_layers: int = N_LAYERS) -> List[bool]:
    """True for a full-context (NoPE) layer.  The pages give the counts (14 full,
    35 window) but not the order; this places two full layers in every group
    of seven.  The order does not change any result: each layer of the stack
    is an independent problem with its own inputs."""
    return [(i % 7) in (3, 6) for i in range(n_layers)]


def make_stack(L: int, n_layers: int = N_LAYERS, workload: int = W_STACK_100K,
               full_capacity: Optional[int] = None, fp8: bool = False) -> List[Layer]:
    """49-layer stack for one token at context L: window layers with RoPE on
    513-slot rings, full NoPE layers on contiguous caches (E4M3 caches if fp8)."""
    out = []
    for i, full in enumerate(layer_kinds(n_layers)):
        if full:
            out.append(make_layer(workload, i, L, 0, False, ring=False,
                                  capacity=full_capacity, fp8=fp8))
        else:
            out.append(make_layer(workload, i, L, WINDOW, True, ring=True, fp8=fp8))
    return out


@dataclasses.dataclass
class DecodeInputs:
    """Already-normed q over a contiguous cache (no append)."""
    q: torch.Tensor          # bf16 [B,32,128]
    k_cache: torch.Tensor    # bf16 [B,cap,4,128], or uint8 E4M3 codes
    v_cache: torch.Tensor
    sinks: torch.Tensor      # f32 [32]
    seq_lens: List[int]
    k_scale: Optional[List[float]] = None
    v_scale: Optional[List[float]] = None


def make_decode(L: int, workload: int = W_FULL_100K, B: int = 1,
                capacity: Optional[int] = None, fp8: bool = False) -> DecodeInputs:
    cap = capacity if capacity is not None else L
    k = bf16_normal((B, cap, NUM_KV_HEADS, HEAD_DIM), seed_for(workload, 0, _T_KC))
    v = bf16_normal((B, cap, NUM_KV_HEADS, HEAD_DIM), seed_for(workload, 0, _T_VC))
    ks = vs = None
    if fp8:
        ks, vs = fp8_scales(seed_for(workload, 0, _T_KS)), fp8_scales(seed_for(workload, 0, _T_VS))
        k, v = to_e4m3_codes(k, ks), to_e4m3_codes(v, vs)
    return DecodeInputs(
        q=bf16_normal((B, NUM_Q_HEADS, HEAD_DIM), seed_for(workload, 0, _T_Q)),
        k_cache=k, v_cache=v,
        sinks=f32_normal((NUM_Q_HEADS,), seed_for(workload, 0, _T_SINK)),
        seq_lens=[L] * B, k_scale=ks, v_scale=vs)


@dataclasses.dataclass
class PagedBatch:
    q: torch.Tensor            # bf16 [B,32,128]
    k_pool: torch.Tensor       # bf16 [num_blocks,64,4,128]
    v_pool: torch.Tensor
    block_table: torch.Tensor  # int32 [B,max_blocks]
    seq_lens: List[int]
    sinks: torch.Tensor        # f32 [32] (shared by all requests)
    k_scale: Optional[List[float]] = None   # E4M3 pools
    v_scale: Optional[List[float]] = None


def log_uniform_lengths(B: int, lo: int, hi: int, seed: int) -> List[int]:
    g = _gen(seed)
    u = torch.rand((B,), generator=g, dtype=torch.float64)
    return [int(round(math.exp(math.log(lo) + float(x) * (math.log(hi) - math.log(lo)))))
            for x in u]


def make_paged_batch(B: int = 32, lo: int = 4096, hi: int = 131072,
                     workload: int = W_PAGED_BATCH, spare_blocks: int = 0,
                     seq_lens: Optional[List[int]] = None, fp8: bool = False) -> PagedBatch:
    """Requests with log-uniform lengths in [lo, hi]; each request's blocks are
    drawn from one randomly permuted pool (block ids shuffled)."""
    if seq_lens is None:
        seq_lens = log_uniform_lengths(B, lo, hi, seed_for(workload, 0, 100))
    B = len(seq_lens)
    nblk = [-(-L // BLOCK_SIZE) for L in seq_lens]
    num_blocks = sum(nblk) + spare_blocks
    perm = torch.randperm(num_blocks, generator=_gen(seed_for(workload, 0, 101)))
    max_blocks = max(nblk)
    table = torch.zeros((B, max_blocks), dtype=torch.int32)
    k = 0
    for b, n in enumerate(nblk):
        table[b, :n] = perm[k:k + n].to(torch.int32)
        k += n
    k = bf16_normal((num_blocks, BLOCK_SIZE, NUM_KV_HEADS, HEAD_DIM), seed_for(workload, 0, _T_KC))
    v = bf16_normal((num_blocks, BLOCK_SIZE, NUM_KV_HEADS, HEAD_DIM), seed_for(workload, 0, _T_VC))
    ks = vs = None
    if fp8:
        ks, vs = fp8_scales(seed_for(workload, 0, _T_KS)), fp8_scales(seed_for(workload, 0, _T_VS))
        k, v = to_e4m3_codes(k, ks), to_e4m3_codes(v, vs)
    return PagedBatch(
        q=bf16_normal((B, NUM_Q_HEADS, HEAD_DIM), seed_for(workload, 0, _T_Q)),
        k_pool=k, v_pool=v, block_table=table, seq_lens=list(seq_lens),
        sinks=f32_normal((NUM_Q_HEADS,), seed_for(workload, 0, _T_SINK)),
        k_scale=ks, v_scale=vs)


@dataclasses.dataclass
class PrefillInputs:
    """The raw activations of one layer for a T-token prompt."""
    q_raw: torch.Tensor        # bf16 [T,32,128]
    k_raw: torch.Tensor        # bf16 [T,4,128]
    v_raw: torch.Tensor        # bf16 [T,4,128]
    w_q: torch.Tensor          # bf16 [128]
    w_k: torch.Tensor          # bf16 [128]
    sinks: torch.Tensor        # f32 [32]
    window: int
    rope: bool


def make_prefill(T: int, window: int, workload: int = W_PREFILL, layer: int = 0) -> PrefillInputs:
    """A prompt of T tokens for one layer (window 513 with RoPE, or 0 without),
    with the value distributions of make_layer."""
    s = lambda t: seed_for(workload, layer, t)  # noqa: E731
    return PrefillInputs(
        q_raw=bf16_normal((T, NUM_Q_HEADS, HEAD_DIM), s(_T_Q)),
        k_raw=bf16_normal((T, NUM_KV_HEADS, HEAD_DIM), s(_T_K)),
        v_raw=bf16_normal((T, NUM_KV_HEADS, HEAD_DIM), s(_T_V)),
        w_q=bf16_normal((HEAD_DIM,), s(_T_WQ), 1.0, 0.1),
        w_k=bf16_normal((HEAD_DIM,), s(_T_WK), 1.0, 0.1),
        sinks=f32_normal((NUM_Q_HEADS,), s(_T_SINK)),
        window=window, rope=window > 0)
