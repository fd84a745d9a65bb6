"""Device memory of the library grows linearly in the sequence length.

The pages claim that ring attention needs memory linear in the sequence
length ("RingAttention核心功能全解析", 实战价值 2), instead of the quadratic
score matrix.  Here: the library allocates no device memory of its own (all
of it comes from the caller; the free memory not held by torch's caching
allocator does not move across the calls), and what the caller allocates
for a forward + backward (outputs plus the declared workspaces) is linear in
S at a fixed per-token constant.
"""

from __future__ import annotations

import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu
ra = pytest.importorskip("long_context_exact_ordered_b200")


def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def _outside_torch():
    """Bytes of device memory in use by anything other than torch's allocator."""
    free, total = torch.cuda.mem_get_info()
    return total - free - torch.cuda.memory_reserved()


@pytest.mark.parametrize("segments", [None, "packed"])
def test_memory_is_linear_in_sequence_length(segments):
    B, H, D, P = 1, 4, 128, 8
    per_token = []
    # the first launches load the module and size the context's local memory:
    # warm up with the same kernels before measuring
    for S in (8192, 8192, 16384, 32768):
        w = W.small_workload(B=B, H=H, D=D, S=S, P=P, chunk=512, causal_block_size=1, segments=segments, seed=61,
                             doc_lo=1024, doc_hi=4096, backward=True)
        inp = W.make_inputs(w, dev())
        kw = dict(query_chunk_size=512, key_chunk_size=512, causal_block_size=1, ring_size=P)
        p = ra.api._params(S, 512, 512, 1, P, None)
        ws_f = ra.workspace_size(0, inp["q"], p, False, inp["seg"] is not None)
        ws_b = ra.workspace_size(1, inp["q"], p, False, inp["seg"] is not None)
        torch.cuda.synchronize()
        outside0 = _outside_torch()
        torch.cuda.reset_peak_memory_stats()
        if len(per_token) == 0:
            outside0 = None          # warm-up pass
        base = torch.cuda.memory_allocated()
        o, lse = ra.ringattention(inp["q"], inp["k"], inp["v"], None, inp["seg"], **kw)
        dq, dk, dv = ra.ringattention_backward(inp["q"], inp["k"], inp["v"], o, lse, inp["do"], None, inp["seg"],
                                               **kw)
        torch.cuda.synchronize()
        assert ra.device_status() == 0
        peak = torch.cuda.max_memory_allocated() - base
        outside1 = _outside_torch()
        # the library itself allocated nothing (any cudaMalloc of its own would show here)
        assert outside0 is None or outside1 == outside0
        # the caller's allocations: o, lse, dq, dk, dv and the larger of the two workspaces
        # (each is released when its call returns); torch's caching allocator may hand
        # out a cached block up to 1 MiB larger than asked without splitting it
        declared = sum(t.numel() * t.element_size() for t in (o, lse, dq, dk, dv)) + max(ws_f, ws_b)
        assert peak <= declared + 6 * (1 << 20)
        # workspaces are linear in S: metadata, Delta / lse rows and the fp32 dQ accumulator
        per_token.append((declared, S, ws_b))
        del o, lse, dq, dk, dv, inp        # the next size starts from the same base
        torch.cuda.synchronize()
    per_token = per_token[1:]
    for dec, S, ws in per_token[1:]:
        d0, S0, w0 = per_token[0]
        assert abs(dec / S - d0 / S0) <= 0.01 * d0 / S0
        assert abs(ws / S - w0 / S0) <= 0.01 * w0 / S0
    # and far below a quadratic score matrix (one head's fp32 S x S at the largest S)
    assert per_token[-1][0] < 32768 * 32768 * 4


def test_ring_step_allocates_nothing():
    w = W.small_workload(B=1, H=2, D=128, S=2048, P=2, chunk=1024, causal_block_size=1, seed=62)
    inp = W.make_inputs(w, dev())
    acc, m, l = ra.init_state(1, 1024, 2, 128, dev())
    q, k, v = inp["q"], inp["k"], inp["v"]
    ra.ring_step(q[:, 1024:], k[:, :1024], v[:, :1024], 1024, 0, acc, m, l, causal_block_size=1)   # warm-up
    torch.cuda.synchronize()
    outside0 = _outside_torch()
    base = torch.cuda.memory_allocated()
    ra.ring_step(q[:, 1024:], k[:, :1024], v[:, :1024], 1024, 0, acc, m, l, causal_block_size=1)
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated() == base
    assert _outside_torch() == outside0
