"""KV-cache ring steps (long_context_exact_ordered_b200.kvcache) on CPU.

The cache's block walk, causal cut-off, prefix chain and global positions are
checked with the oracle's online step in float64 standing in for ra_step
(the GPU test runs the same scenario on the tensor cores).
"""

from __future__ import annotations

import pytest
import torch

from kvcache_case import max_errors, run_case
from long_context_exact_ordered_b200.kvcache import KVCache
from oracle_steps import oracle_finalize, oracle_step


@pytest.mark.parametrize("block", [7, 16, 1000])
def test_kvcache_chunks_equal_full_causal_attention(block):
    H, D = 2, 16

    def make(batch, prefix):
        return KVCache(batch, H, D, capacity=128, block=block, dtype=torch.float64, device="cpu", prefix=prefix)

    res = run_case(make, torch.float64, "cpu", H, D, n_prefix=40, prefix_chunks=(25, 15), chunks=(17, 30, 1),
                   step=oracle_step, finalize=oracle_finalize)
    eo, el = max_errors(res)
    assert eo < 1e-6 and el < 1e-6, (eo, el)       # fp32 running state, float64 arithmetic


def test_kvcache_rejects_bad_prefix_and_overflow():
    p = KVCache(2, 2, 16, capacity=8, dtype=torch.float64, device="cpu")
    with pytest.raises(ValueError):
        KVCache(3, 2, 16, capacity=8, dtype=torch.float64, device="cpu", prefix=p)
    c = KVCache(1, 2, 16, capacity=8, dtype=torch.float64, device="cpu")
    with pytest.raises(ValueError):
        c.append(torch.zeros(1, 9, 2, 16, dtype=torch.float64), torch.zeros(1, 9, 2, 16, dtype=torch.float64))
