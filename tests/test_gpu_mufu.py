"""MUFU exp2 throughput on this B200, the forward's second ceiling (one ex2 per
visible pair next to 4*D flop of MMAs), measured by the debug build's
microbenchmark and held to a plausible range.  Run with -s to see the rate."""

from __future__ import annotations

import pytest
import torch

pytestmark = pytest.mark.gpu
ra = pytest.importorskip("long_context_exact_ordered_b200")


def test_mufu_ex2_rate():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_exact_ordered_b200 import _lib

    dbg = _lib.load_count()
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    cycles = torch.zeros(sms, dtype=torch.int64, device="cuda")
    sink = torch.zeros(512, dtype=torch.float32, device="cuda")
    iters = 4096
    s = torch.cuda.current_stream().cuda_stream
    assert dbg.ra_debug_ex2_rate(iters, sms, cycles.data_ptr(), sink.data_ptr(), s) == 0   # warm-up
    assert dbg.ra_debug_ex2_rate(iters, sms, cycles.data_ptr(), sink.data_ptr(), s) == 0
    torch.cuda.synchronize()
    rate = 512 * 8 * iters / cycles.double().mean().item()
    print(f"MUFU ex2 per clock per SM: {rate:.2f}")
    assert 4.0 <= rate <= 64.0
