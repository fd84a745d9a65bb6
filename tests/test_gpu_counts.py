"""Mask bit-exactness of the tensor-core kernels (needs a B200).

The debug build of the library (-DRA_DEBUG_COUNT, include/ringattn_debug.h)
makes the forward kernel count, for each query row, the keys its own tile
skipping and per-element masking let into the softmax, and the backward
kernel count, for each key, the query rows it is paired with.  Those integer
counts must equal the oracle's integer mask bit for bit: row sums
(visible_count_rows) for the forward, column sums (visible_count_cols) for
the backward.  Which pairs take part is fixed by the pages' mask arguments
("RingAttention核心功能全解析", 核心API调用: causal_block_size, segment_ids,
attention_bias); completeness over them by "手把手拆解RingAttention…" §1.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads as W

pytestmark = pytest.mark.gpu
ra = pytest.importorskip("long_context_exact_ordered_b200")


def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def make(D, S, P, c, segments, bias, B=2, H=2, seed=31):
    w = W.small_workload(B=B, H=H, D=D, S=S, P=P, chunk=S // P, causal_block_size=c, segments=segments,
                         seed=seed, doc_lo=40, doc_hi=600, backward=True)
    inp = W.make_inputs(w, dev())
    if bias == "neginf":
        g = torch.Generator(device="cpu").manual_seed(seed + 1)
        b = 0.5 * torch.randn((B, S), generator=g)
        b[:, torch.randint(0, S, (S // 7,), generator=g)] = float("-inf")
        b[:, 0] = float("-inf")          # with causal masking, query row 0 then sees no key at all
        inp["bias"] = b.to(dev())
    return w, inp


CASES = [
    # D, S, P, causal_block_size, segments, bias, ring_order
    (128, 1024, 4, 1, None, None, None),
    (128, 1024, 2, None, "packed", None, None),
    (128, 1536, 3, 1, "packed", "neginf", None),
    (128, 1024, 4, 3, None, None, None),
    (128, 1024, 4, 200, None, "neginf", None),
    (128, 1024, 4, 1, "packed", None, [2, 0, 3, 1]),
    (128, 1024, 1, None, None, "neginf", None),
    (64, 1024, 4, 1, "packed", "neginf", None),
    (64, 2048, 8, 5, None, None, [7, 6, 5, 4, 3, 2, 1, 0]),
    (128, 1000, 2, 1, "packed", "neginf", None),        # ragged last tile (1000 = 7 * 128 + 104)
    (128, 1000, 4, None, None, None, [1, 3, 0, 2]),
    (64, 1000, 4, 3, "packed", None, None),
]


def _host(t):
    return None if t is None else t.cpu().numpy()


def _expect(w, inp, cols):
    seg = _host(inp["seg"])
    bias = None if inp["bias"] is None else inp["bias"].double().cpu().numpy()
    out = np.zeros((w.B, w.H, w.S), dtype=np.int64)
    for b in range(w.B):
        sb = None if seg is None else seg[b]
        bb = None if bias is None else bias[b]
        if cols:
            cnt = oracle.visible_count_cols(w.S, w.causal_block_size, sb, bb)
        else:
            cnt = oracle.visible_count_rows(np.arange(w.S), w.S, w.causal_block_size, sb, bb)
        out[b, :, :] = cnt[None, :]
    return out


@pytest.mark.parametrize("D,S,P,c,segments,bias,order", CASES)
def test_forward_counts_match_integer_mask(D, S, P, c, segments, bias, order):
    w, inp = make(D, S, P, c, segments, bias)
    rows = torch.full((w.B, w.H, w.S), -1, dtype=torch.int32, device=dev())
    kw = dict(query_chunk_size=w.chunk, key_chunk_size=w.chunk, causal_block_size=c, ring_size=P, ring_order=order)
    with ra.visible_count_probe(fwd_row_counts=rows):
        ra.ringattention(inp["q"], inp["k"], inp["v"], inp["bias"], inp["seg"], **kw)
    torch.cuda.synchronize()
    assert ra.device_status() == 0
    np.testing.assert_array_equal(rows.cpu().numpy().astype(np.int64), _expect(w, inp, cols=False))


@pytest.mark.parametrize("D,S,P,c,segments,bias,order", CASES)
def test_backward_counts_match_integer_mask(D, S, P, c, segments, bias, order):
    w, inp = make(D, S, P, c, segments, bias)
    kw = dict(query_chunk_size=w.chunk, key_chunk_size=w.chunk, causal_block_size=c, ring_size=P, ring_order=order)
    o, lse = ra.ringattention(inp["q"], inp["k"], inp["v"], inp["bias"], inp["seg"], **kw)
    cols = torch.zeros((w.B, w.H, w.S), dtype=torch.int32, device=dev())
    with ra.visible_count_probe(bwd_col_counts=cols):
        ra.ringattention_backward(inp["q"], inp["k"], inp["v"], o, lse, inp["do"], inp["bias"], inp["seg"], **kw)
    torch.cuda.synchronize()
    assert ra.device_status() == 0
    np.testing.assert_array_equal(cols.cpu().numpy().astype(np.int64), _expect(w, inp, cols=True))


def test_counts_at_many_tiles():
    """A packed causal case over 64 key tiles per head, both directions."""
    w, inp = make(128, 8192, 8, 1, "packed", None, B=1, H=2, seed=33)
    kw = dict(query_chunk_size=w.chunk, key_chunk_size=w.chunk, causal_block_size=1, ring_size=w.P)
    rows = torch.full((w.B, w.H, w.S), -1, dtype=torch.int32, device=dev())
    cols = torch.zeros((w.B, w.H, w.S), dtype=torch.int32, device=dev())
    with ra.visible_count_probe(fwd_row_counts=rows, bwd_col_counts=cols):
        o, lse = ra.ringattention(inp["q"], inp["k"], inp["v"], None, inp["seg"], **kw)
        ra.ringattention_backward(inp["q"], inp["k"], inp["v"], o, lse, inp["do"], None, inp["seg"], **kw)
    torch.cuda.synchronize()
    assert ra.device_status() == 0
    np.testing.assert_array_equal(rows.cpu().numpy().astype(np.int64), _expect(w, inp, cols=False))
    np.testing.assert_array_equal(cols.cpu().numpy().astype(np.int64), _expect(w, inp, cols=True))


def test_release_build_is_restored():
    """After the probe block, calls go to the release library again."""
    from long_context_exact_ordered_b200 import _lib

    rel = _lib.load()
    rows = torch.zeros((1, 1, 256), dtype=torch.int32, device=dev())
    with ra.visible_count_probe(fwd_row_counts=rows):
        assert _lib.load() is _lib.load_count()
    assert _lib.load() is rel
