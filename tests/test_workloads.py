"""The seeded input generators (no GPU)."""

import numpy as np
import torch

import workloads as W


def test_packed_segments_cover_and_respect_length_range():
    seg = W.packed_segment_ids(131072, 1003)
    assert seg.shape == (131072,) and seg.dtype == np.int32
    _, lengths = np.unique(seg, return_counts=True)
    assert lengths.sum() == 131072
    assert np.all(lengths[:-1] >= 1024) and np.all(lengths[:-1] <= 32768)
    assert 1 <= lengths[-1] <= 32768
    assert np.all(np.diff(seg) >= 0)                      # documents are contiguous runs


def test_make_inputs_is_seeded_and_shaped():
    w = W.small_workload(B=2, H=3, D=64, S=256, P=2, dtype="bf16", segments="packed", doc_lo=10, doc_hi=50,
                         backward=True)
    a = W.make_inputs(w)
    b = W.make_inputs(w)
    for name in ("q", "k", "v", "do"):
        assert a[name].shape == (2, 256, 3, 64) and a[name].dtype == torch.bfloat16
        assert torch.equal(a[name], b[name])
    assert a["seg"].shape == (2, 256) and a["seg"].dtype == torch.int32
    assert not torch.equal(a["q"], a["k"])


def test_sample_rows_distinct_and_cover_edges():
    w = W.WORKLOADS["packed128k"]
    seg = W.packed_segment_ids(w.S, w.seed)[None]
    s = W.sample_rows(w, seg)
    assert s.shape == (4096, 3)
    assert len({tuple(r) for r in s}) == 4096
    rows = set(s[:, 2].tolist())
    blk = w.S // w.P
    for r in range(w.P):
        assert r * blk in rows and (r + 1) * blk - 1 in rows
    starts = np.nonzero(np.r_[True, seg[0][1:] != seg[0][:-1]])[0]
    assert set(starts.tolist()) <= rows
    assert s[:, 0].max() < w.B and s[:, 1].max() < w.H and s[:, 2].max() < w.S
