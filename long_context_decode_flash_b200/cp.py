"""Context-parallel decode of a full-context layer across ranks, one process
per GPU: every rank holds a contiguous range of the layer's tokens in its own
cache, runs the split-KV attention of the (replicated) query over it
(flint_attn_decode_partial), the ranks all-gather their partials (32 x (128 +
2) fp32 per request, over NCCL on GPUs), and every rank merges them with the
sinks (flint_merge_partials).  The arithmetic is the split-KV decode of one
GPU, cut at rank boundaries; the pages serve on one GPU, so this is the
multi-GPU reading of it for contexts beyond one GPU's memory.

This module only marshals: both compute steps run in the CUDA library."""
from __future__ import annotations

from typing import List, Sequence, Tuple

import torch
import torch.distributed as dist

from . import flint


def rank_ranges(L: int, world: int) -> List[Tuple[int, int]]:
    """Token ranges [lo, hi) of a context of L tokens over `world` ranks, in
    rank order, as even as possible (the first L % world ranks hold one more)."""
    if L < world or world < 1:
        raise ValueError(f"{L} tokens cannot give each of {world} ranks at least one")
    base, extra = divmod(L, world)
    out, lo = [], 0
    for r in range(world):
        hi = lo + base + (1 if r < extra else 0)
        out.append((lo, hi))
        lo = hi
    return out


def gather_partials(part: torch.Tensor, group=None) -> torch.Tensor:
    """All ranks' partials [B, F] stacked in rank order: [world, B, F]; a
    process without a process group is a single rank."""
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    if world == 1:
        return part.unsqueeze(0)
    bufs = [torch.empty_like(part) for _ in range(world)]
    dist.all_gather(bufs, part.contiguous(), group=group)
    return torch.stack(bufs)


def cp_decode(q: torch.Tensor, local_cache: flint.KVCache, local_lens: Sequence[int], sinks: torch.Tensor,
              out: torch.Tensor, ws: torch.Tensor, group=None, dev_err=None) -> torch.Tensor:
    """One decode step of a full layer whose tokens are spread over the ranks
    of `group`: q [B, 32, 128] (normed, the same on every rank), this rank's
    cache and the number of its tokens per request; out [B, 32, 128] fp32 is
    the same on every rank afterwards."""
    part = torch.empty((len(local_lens), flint.CP_PARTIAL_FLOATS), dtype=torch.float32, device=q.device)
    flint.flint_attn_decode_partial(q, local_cache, local_lens, part, ws, dev_err=dev_err)
    flint.flint_merge_partials(gather_partials(part, group), sinks, out)
    return out
