"""Index checks of the debug build on the paths the tests drive (needs a B200).

The debug build (-DRA_DEBUG_COUNT, include/ringattn_debug.h) tests every
index its kernels compute for a global or shared-memory access against the
extent before the access, skips an out-of-range access and records the first
one (ra_debug_bounds).  The sanitizer tools are not available on the GPU
machines these tests run on; these checks stand in for their out-of-bounds
detection.  Each case runs an entry point through the debug build over
ragged, packed, biased, head-dim-64 and ring-step inputs, then requires that
no index was out of range, that no wait gave up, and that the results are
those of the release build (bit for bit where the release path is
deterministic).
"""

from __future__ import annotations

import contextlib
import ctypes

import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu
ra = pytest.importorskip("long_context_exact_ordered_b200")


def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


@contextlib.contextmanager
def debug_build():
    from long_context_exact_ordered_b200 import _lib

    dbg = _lib.load_count()
    hit = ctypes.c_uint64(0)
    assert dbg.ra_debug_bounds(ctypes.byref(hit)) == 0   # start clean
    prev = _lib.swap(dbg)
    try:
        yield
    finally:
        _lib.swap(prev)
    torch.cuda.synchronize()
    assert dbg.ra_debug_bounds(ctypes.byref(hit)) == 0
    site, index = hit.value >> 48, hit.value & ((1 << 48) - 1)
    assert hit.value == 0, f"index out of range at site {site} (index {index})"
    assert ra.device_status() == 0


def make(D, S, P, c, segments, bias, B=2, H=2, seed=61):
    w = W.small_workload(B=B, H=H, D=D, S=S, P=P, chunk=S // P, causal_block_size=c, segments=segments,
                         seed=seed, doc_lo=40, doc_hi=400, backward=True)
    inp = W.make_inputs(w, dev())
    if bias == "neginf":
        g = torch.Generator(device="cpu").manual_seed(seed + 1)
        b = torch.randn((B, S), generator=g)
        b[:, torch.randint(0, S, (S // 6,), generator=g)] = float("-inf")
        inp["bias"] = b.to(dev())
    return w, inp


CASES = [
    # D, S, P, causal_block_size, segments, bias
    (128, 1000, 2, 1, "packed", "neginf"),    # ragged last tile
    (64, 1000, 4, 3, "packed", None),
    (128, 1536, 3, None, None, "neginf"),
    (64, 2048, 8, 1, None, None),
    (128, 130, 1, 1, None, None),             # one full tile and two tokens
]


@pytest.mark.parametrize("D,S,P,c,segments,bias", CASES)
def test_forward_backward_indices_in_range(D, S, P, c, segments, bias):
    w, inp = make(D, S, P, c, segments, bias)
    kw = dict(query_chunk_size=w.chunk, key_chunk_size=w.chunk, causal_block_size=c, ring_size=P)
    args = (inp["q"], inp["k"], inp["v"], inp["bias"], inp["seg"])
    o_r, lse_r = ra.ringattention(*args, **kw)
    g_r = ra.ringattention_backward(inp["q"], inp["k"], inp["v"], o_r, lse_r, inp["do"], inp["bias"], inp["seg"],
                                    **kw)
    with debug_build():
        o_d, lse_d = ra.ringattention(*args, **kw)
        g_d = ra.ringattention_backward(inp["q"], inp["k"], inp["v"], o_d, lse_d, inp["do"], inp["bias"],
                                        inp["seg"], **kw)
    torch.cuda.synchronize()
    assert torch.equal(o_d, o_r) and torch.equal(lse_d, lse_r)
    # dK, dV: fixed accumulation order per key tile; dQ: bulk reduce-adds in any order
    assert torch.equal(g_d[1], g_r[1]) and torch.equal(g_d[2], g_r[2])
    assert (g_d[0].float() - g_r[0].float()).abs().max().item() <= 1e-2


@pytest.mark.parametrize("D", [128, 64])
def test_ring_step_indices_in_range(D):
    """Ring steps with segments and a bias, a ragged visiting block, and a
    key/value block of batch 1 shared by every query row."""
    w, inp = make(D, 1000, 4, 1, "packed", "neginf", B=2, H=2)
    q, k, v, seg, bias = inp["q"], inp["k"], inp["v"], inp["seg"], inp["bias"]
    outs = []
    for lib_ctx in (contextlib.nullcontext(), debug_build()):
        with lib_ctx:
            acc, m, l = ra.init_state(2, 250, 2, D, q.device)
            for ks in (slice(0, 250), slice(250, 500), slice(500, 750), slice(750, 1000)):
                ra.ring_step(q[:, 500:750], k[:, ks], v[:, ks], 500, ks.start, acc, m, l, bias_blk=bias[:, ks],
                             seg_q=seg[:, 500:750].contiguous(), seg_k=seg[:, ks].contiguous(),
                             causal_block_size=1)
            ra.ring_step(q[:, 500:750], k[:1, 0:250], v[:1, 0:250], 500, 0, acc, m, l, causal_block_size=1)
            o, lse = ra.finalize(acc, m, l)
            o2, lse2 = ra.lse_merge(o, lse, o, lse)
        torch.cuda.synchronize()
        outs.append((o, lse, o2, lse2))
    for a, b in zip(*outs):
        assert torch.equal(a, b)


def test_feedforward_indices_in_range():
    g = torch.Generator(device="cpu").manual_seed(5)
    T, dm, dff = 1000, 256, 384
    x = (torch.randn(T, dm, generator=g) * 0.5).to(torch.bfloat16).to(dev())
    w1, w3 = ((torch.randn(dff, dm, generator=g) * dm ** -0.5).to(torch.bfloat16).to(dev()) for _ in range(2))
    w2 = (torch.randn(dm, dff, generator=g) * dff ** -0.5).to(torch.bfloat16).to(dev())
    y_r = ra.blockwise_feedforward(x, w1, w3, w2, chunk_size=384)
    with debug_build():
        y_d = ra.blockwise_feedforward(x, w1, w3, w2, chunk_size=384)
    torch.cuda.synchronize()
    assert torch.equal(y_d, y_r)


def test_static_forward_indices_in_range():
    w, inp = make(128, 1000, 2, 1, "packed", "neginf", B=1, H=2)
    kw = dict(query_chunk_size=w.chunk, key_chunk_size=w.chunk, causal_block_size=1, ring_size=2)
    o_r, lse_r = ra.ringattention_static(inp["q"], inp["k"], inp["v"], inp["bias"], inp["seg"], **kw)
    with debug_build():
        o_d, lse_d = ra.ringattention_static(inp["q"], inp["k"], inp["v"], inp["bias"], inp["seg"], **kw)
    torch.cuda.synchronize()
    assert torch.equal(o_d, o_r) and torch.equal(lse_d, lse_r)
