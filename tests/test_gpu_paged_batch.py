"""Batched paged decode at its full size: 32 requests with context lengths
log-uniform in [4096, 131072], bf16 KV in 64-token blocks behind a randomly
permuted block table, shared sinks; once as full-context layers and once as
sliding-window layers.  Launched as the benchmark launches it; the oracle
checks a sample of requests (every head)."""
import numpy as np
import pytest
import torch

import oracle
from long_context_decode_flash_b200 import flint
from long_context_decode_flash_b200 import inputs as I

from helpers import dev, parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def batch():
    pb = I.make_paged_batch()
    d = dict(q=dev(pb.q), k=dev(pb.k_pool), v=dev(pb.v_pool), table=dev(pb.block_table),
             sinks=dev(pb.sinks))
    return pb, d


@pytest.mark.parametrize("window", [0, 513])
def test_paged_batch_32_requests(batch, window):
    pb, d = batch
    B = len(pb.seq_lens)
    assert B == 32 and min(pb.seq_lens) >= 4096 and max(pb.seq_lens) <= 131072
    cache = flint.kv_cache(d["k"], d["v"], flint.PAGED, block_table=d["table"],
                           num_blocks=pb.k_pool.shape[0])
    out = torch.full((B, 32, 128), float("nan"), dtype=torch.float32, device="cuda")
    ws = flint.workspace(B)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    flint.flint_attn_decode(d["q"], cache, pb.seq_lens, d["sinks"], window, out, ws, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    got = out.cpu().numpy()
    assert np.isfinite(got).all()
    kp, vp = I.bits(pb.k_pool), I.bits(pb.v_pool)
    for b in range(B):  # every request (~1.1M tokens of oracle work, ~8 s)
        want = oracle.attn_decode(I.bits(pb.q[b]), kp, vp, pb.seq_lens[b],
                                  pb.sinks.numpy().astype(np.float64), window,
                                  layout=oracle.PAGED, block_table=pb.block_table[b].numpy())
        parity(got[b], want, f"request {b} L={pb.seq_lens[b]} window={window}")
