"""Device-side failure detection, exercised without any GPU fault.

A kernel waits, through the attention kernels' own bounded mbarrier wait, on a
barrier phase that nothing completes; the wait must give up, record
RA_ERR_DEVICE_TIMEOUT in the status word and return, leaving the context
usable: the next attention call works and reports a clean status.
"""

import pytest
import torch

import workloads as W
from checker import compare
from gpu_util import oracle_full, to64

pytestmark = pytest.mark.gpu
ra = pytest.importorskip("long_context_exact_ordered_b200")


def test_bounded_wait_gives_up_and_reports_timeout():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    assert ra.device_status() == 0
    assert ra.selftest_timeout(2_000_000) == 9          # RA_ERR_DEVICE_TIMEOUT, read and cleared
    assert ra.device_status() == 0                      # cleared by the read
    w = W.small_workload(B=1, H=2, D=128, S=512, P=2, chunk=256, causal_block_size=1, seed=41)
    inp = W.make_inputs(w, torch.device("cuda:0"))
    o, lse = ra.ringattention(inp["q"], inp["k"], inp["v"], None, None, query_chunk_size=256,
                              key_chunk_size=256, causal_block_size=1, ring_size=2)
    assert ra.device_status() == 0
    ro, rl = oracle_full(inp, 1)
    assert compare(to64(o), ro, "bf16").ok
