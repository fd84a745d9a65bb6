"""The plain definition of masked softmax attention, float64 (the oracle).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

What the method computes.  Ring Attention claims to keep *global* attention
complete while cutting the sequence into blocks ([RA-LWM] §1, complexity
table row "RingAttention ... 完整保留", and the note that the blocks together
form the complete attention map).  So its result is exactly full softmax
attention, and this module is that definition written out, row by row:

    scale        = 1 / sqrt(D)
    visible(i,j) = causal_ok(i,j) and seg[i] == seg[j] and bias[j] > -inf
    causal_ok    = (i // c) >= (j // c)   if causal_block_size c >= 1, else True
    s_ij         = scale * <q_i, k_j> + bias[j]          (visible pairs only)
    lse_i        = log sum_j exp(s_ij)                    (-inf if none visible)
    o_i          = sum_j exp(s_ij - lse_i) v_j            (0 if none visible)

Backward (the recompute policy of [RA-core] 核心API调用 saves nothing but
the per-row log-sum-exp; the gradient itself is the analytic derivative of
the definition above, given an upstream dO):

    Dl_i  = <dO_i, o_i>
    P_ij  = exp(s_ij - lse_i)
    dP_ij = <dO_i, v_j>
    dS_ij = P_ij (dP_ij - Dl_i)
    dQ_i  = scale sum_j dS_ij k_j
    dK_j  = scale sum_i dS_ij q_i
    dV_j  = sum_i P_ij dO_i

Readings where the pages are silent (each listed in the design notes):
* ``causal_block_size`` (named in [RA-core] 核心技术原理 1, "=1 enables
  causal attention"): key j is visible to query i iff floor(i/c) >= floor(j/c);
  None or 0 means non-causal.  Positions are global token indices.
* ``attention_bias`` (named in [RA-core] 核心API调用): additive float bias per
  key, shape [B, S], broadcast over heads and queries; -inf masks the key.
* ``segment_ids`` (named in [RA-core] 核心API调用): int [B, S]; a key is
  visible only to queries carrying the same id.
* The softmax scale is 1/sqrt(D).
* A row with no visible key has o = 0 and lse = -inf (and zero gradients).

Layouts: q, k, v, o, dO are [B, S, H, D] (batch, sequence, heads, head dim,
the sequence-sharded order of the pages' shard_map spec in [RA-core]
核心技术原理 3); lse is [B, H, S].

Evaluation is row-chunked (each chunk of query rows is the definition applied
to those rows; no key blocking, no merging).
"""

from __future__ import annotations

import math

import numpy as np

_ROW_CHUNK_ELEMS = 1 << 25  # score-matrix elements evaluated at once (256 MiB fp64)


def _f64(x):
    return np.asarray(x, dtype=np.float64)


def causal_ok(i, j, causal_block_size):
    """Causal visibility of key position(s) j from query position(s) i.

    ``causal_block_size`` c: None/0 -> everything visible; c >= 1 ->
    visible iff i // c >= j // c (c = 1 is ordinary causal attention).
    Broadcasts like numpy.
    """
    i = np.asarray(i, dtype=np.int64)
    j = np.asarray(j, dtype=np.int64)
    if not causal_block_size:
        return np.ones(np.broadcast(i, j).shape, dtype=bool)
    c = int(causal_block_size)
    return (i // c) >= (j // c)


def visible_mask(rows, S, causal_block_size=None, seg_b=None, bias_b=None, keys=None):
    """Boolean visibility [len(rows), len(keys)] for query rows ``rows`` of one
    batch against key positions ``keys`` (default: all S keys).

    ``seg_b`` / ``bias_b`` are that batch's segment ids / bias ([S]) or None.
    """
    rows = np.asarray(rows, dtype=np.int64)
    keys = np.arange(S, dtype=np.int64) if keys is None else np.asarray(keys, dtype=np.int64)
    vis = causal_ok(rows[:, None], keys[None, :], causal_block_size)
    if seg_b is not None:
        seg_b = np.asarray(seg_b)
        vis = vis & (seg_b[rows][:, None] == seg_b[keys][None, :])
    if bias_b is not None:
        vis = vis & (np.asarray(bias_b, dtype=np.float64)[keys][None, :] > -np.inf)
    return vis


def _rows_forward(q_rows, k_h, v_h, rows, causal_block_size, seg_b, bias_b):
    """Definition applied to query rows ``rows`` of one (b, h).

    q_rows [n, D], k_h / v_h [S, D] float64.  Returns o [n, D], lse [n].
    """
    S, D = k_h.shape
    scale = 1.0 / math.sqrt(D)
    vis = visible_mask(rows, S, causal_block_size, seg_b, bias_b)
    s = scale * (q_rows @ k_h.T)
    if bias_b is not None:
        b = np.where(np.isfinite(bias_b), bias_b, 0.0)  # -inf keys are masked below
        s = s + b[None, :]
    s = np.where(vis, s, -np.inf)
    m = s.max(axis=1)
    any_vis = vis.any(axis=1)
    m_safe = np.where(any_vis, m, 0.0)
    e = np.where(vis, np.exp(s - m_safe[:, None]), 0.0)
    l = e.sum(axis=1)
    lse = np.where(any_vis, m_safe + np.log(np.where(any_vis, l, 1.0)), -np.inf)
    o = np.where(any_vis[:, None], (e @ v_h) / np.where(any_vis, l, 1.0)[:, None], 0.0)
    return o, lse


def _row_chunks(n, S):
    step = max(1, min(n, _ROW_CHUNK_ELEMS // max(S, 1)))
    for a in range(0, n, step):
        yield a, min(n, a + step)


def attention_forward(q, k, v, attention_bias=None, segment_ids=None, causal_block_size=None):
    """Full forward: returns o [B,S,H,D] and lse [B,H,S], float64."""
    q = np.asarray(q)
    B, S, H, D = q.shape
    o = np.zeros((B, S, H, D), dtype=np.float64)
    lse = np.full((B, H, S), -np.inf, dtype=np.float64)
    for b in range(B):
        seg_b = None if segment_ids is None else np.asarray(segment_ids)[b]
        bias_b = None if attention_bias is None else _f64(attention_bias)[b]
        for h in range(H):
            qh, kh, vh = _f64(q[b, :, h, :]), _f64(k[b, :, h, :]), _f64(v[b, :, h, :])
            for a, e in _row_chunks(S, S):
                rows = np.arange(a, e)
                o[b, a:e, h, :], lse[b, h, a:e] = _rows_forward(
                    qh[a:e], kh, vh, rows, causal_block_size, seg_b, bias_b)
    return o, lse


def attention_rows(q, k, v, samples, attention_bias=None, segment_ids=None, causal_block_size=None,
                   q_rows=None):
    """Forward for selected rows only.

    ``samples`` is an int array [n, 3] of (b, h, i).  Returns o [n, D] and
    lse [n] in the order given.  Each (b, h) head's K and V are upcast once
    and all of its sampled rows are evaluated together.  ``q_rows`` [n, D]
    optionally supplies the sampled query vectors directly (then ``q`` is
    not read), so a caller need not hold the whole query tensor.
    """
    samples = np.asarray(samples, dtype=np.int64).reshape(-1, 3)
    D = np.asarray(k).shape[-1]
    S = np.asarray(k).shape[1]
    o = np.zeros((len(samples), D), dtype=np.float64)
    lse = np.zeros(len(samples), dtype=np.float64)
    keys = samples[:, 0] * (1 << 20) + samples[:, 1]
    for key in np.unique(keys):
        idx = np.nonzero(keys == key)[0]
        b, h = int(samples[idx[0], 0]), int(samples[idx[0], 1])
        rows = samples[idx, 2]
        kh, vh = _f64(k[b, :, h, :]), _f64(v[b, :, h, :])
        seg_b = None if segment_ids is None else np.asarray(segment_ids)[b]
        bias_b = None if attention_bias is None else _f64(attention_bias)[b]
        qr = _f64(np.asarray(q)[b, rows, h, :]) if q_rows is None else _f64(np.asarray(q_rows)[idx])
        for a, e in _row_chunks(len(rows), S):
            o[idx[a:e]], lse[idx[a:e]] = _rows_forward(
                qr[a:e], kh, vh, rows[a:e], causal_block_size, seg_b, bias_b)
    return o, lse


def _head_backward(qh, kh, vh, doh, oh, lse_h, rows_all, causal_block_size, seg_b, bias_b,
                   want_dkdv=True):
    """Backward of one (b, h) over query rows ``rows_all``.

    Returns dq [n, D] for those rows and, if ``want_dkdv``, the contributions
    of those rows to dk, dv [S, D].
    """
    S, D = kh.shape
    scale = 1.0 / math.sqrt(D)
    n = len(rows_all)
    dq = np.zeros((n, D), dtype=np.float64)
    dk = np.zeros((S, D), dtype=np.float64) if want_dkdv else None
    dv = np.zeros((S, D), dtype=np.float64) if want_dkdv else None
    for a, e in _row_chunks(n, S):
        rows = rows_all[a:e]
        vis = visible_mask(rows, S, causal_block_size, seg_b, bias_b)
        s = scale * (qh[a:e] @ kh.T)
        if bias_b is not None:
            s = s + np.where(np.isfinite(bias_b), bias_b, 0.0)[None, :]
        lse_r = lse_h[a:e]
        has = np.isfinite(lse_r)
        P = np.where(vis & has[:, None], np.exp(s - np.where(has, lse_r, 0.0)[:, None]), 0.0)
        Dl = np.sum(doh[a:e] * oh[a:e], axis=1)
        dP = doh[a:e] @ vh.T
        dS = P * (dP - Dl[:, None])
        dq[a:e] = scale * (dS @ kh)
        if want_dkdv:
            dk += scale * (dS.T @ qh[a:e])
            dv += P.T @ doh[a:e]
    return dq, dk, dv


def head_backward_cols(qh, kh, vh, doh, oh, lse_h, cols, causal_block_size=None, seg_b=None, bias_b=None):
    """dK and dV of one (b, h) at the key positions ``cols`` only.

    The same sums as the full backward (dK_j = scale * sum_i dS_ij q_i,
    dV_j = sum_i P_ij dO_i over every query row i), restricted to the chosen
    keys, so sampled keys of a long sequence can be checked without the
    whole backward.  ``oh`` / ``lse_h``: the head's forward output (as stored)
    and log-sum-exp for all S rows.
    """
    S, D = kh.shape
    scale = 1.0 / math.sqrt(D)
    cols = np.asarray(cols, dtype=np.int64)
    kc, vc = kh[cols], vh[cols]
    bc = None if bias_b is None else np.where(np.isfinite(bias_b[cols]), bias_b[cols], 0.0)
    dk = np.zeros((len(cols), D), dtype=np.float64)
    dv = np.zeros((len(cols), D), dtype=np.float64)
    for a, e in _row_chunks(S, max(len(cols), 1)):
        rows = np.arange(a, e)
        vis = visible_mask(rows, S, causal_block_size, seg_b, bias_b, keys=cols)
        s = scale * (qh[a:e] @ kc.T)
        if bc is not None:
            s = s + bc[None, :]
        lse_r = lse_h[a:e]
        has = np.isfinite(lse_r)
        P = np.where(vis & has[:, None], np.exp(s - np.where(has, lse_r, 0.0)[:, None]), 0.0)
        Dl = np.sum(doh[a:e] * oh[a:e], axis=1)
        dS = P * (doh[a:e] @ vc.T - Dl[:, None])
        dk += scale * (dS.T @ qh[a:e])
        dv += P.T @ doh[a:e]
    return dk, dv


def attention_backward(q, k, v, do, attention_bias=None, segment_ids=None, causal_block_size=None,
                       o=None, lse=None, heads=None):
    """Analytic backward of the definition.  Returns dq, dk, dv [B,S,H,D] float64.

    ``o`` / ``lse`` default to this module's forward.  ``heads`` optionally
    restricts the work to a list of (b, h) pairs (other heads stay zero).
    """
    q = np.asarray(q)
    B, S, H, D = q.shape
    if o is None or lse is None:
        o, lse = attention_forward(q, k, v, attention_bias, segment_ids, causal_block_size)
    dq = np.zeros((B, S, H, D), dtype=np.float64)
    dk = np.zeros((B, S, H, D), dtype=np.float64)
    dv = np.zeros((B, S, H, D), dtype=np.float64)
    todo = [(b, h) for b in range(B) for h in range(H)] if heads is None else list(heads)
    rows = np.arange(S)
    for b, h in todo:
        seg_b = None if segment_ids is None else np.asarray(segment_ids)[b]
        bias_b = None if attention_bias is None else _f64(attention_bias)[b]
        dq[b, :, h], dk[b, :, h], dv[b, :, h] = _head_backward(
            _f64(q[b, :, h]), _f64(k[b, :, h]), _f64(v[b, :, h]), _f64(do[b, :, h]),
            _f64(o[b, :, h]), _f64(lse[b, h]), rows, causal_block_size, seg_b, bias_b)
    return dq, dk, dv


def attention_backward_rows(q, k, v, do, samples, attention_bias=None, segment_ids=None,
                            causal_block_size=None):
    """dQ for selected rows only (they need only their own o, lse and Dl).

    ``samples`` int [n, 3] of (b, h, i).  Returns dq [n, D] in the order given.
    """
    samples = np.asarray(samples, dtype=np.int64).reshape(-1, 3)
    o_r, lse_r = attention_rows(q, k, v, samples, attention_bias, segment_ids, causal_block_size)
    D = np.asarray(q).shape[-1]
    dq = np.zeros((len(samples), D), dtype=np.float64)
    keys = samples[:, 0] * (1 << 20) + samples[:, 1]
    for key in np.unique(keys):
        idx = np.nonzero(keys == key)[0]
        b, h = int(samples[idx[0], 0]), int(samples[idx[0], 1])
        rows = samples[idx, 2]
        seg_b = None if segment_ids is None else np.asarray(segment_ids)[b]
        bias_b = None if attention_bias is None else _f64(attention_bias)[b]
        dq[idx], _, _ = _head_backward(
            _f64(np.asarray(q)[b, rows, h]), _f64(k[b, :, h]), _f64(v[b, :, h]),
            _f64(np.asarray(do)[b, rows, h]), o_r[idx], lse_r[idx], rows,
            causal_block_size, seg_b, bias_b, want_dkdv=False)
    return dq


def backward_term_magnitudes(q, k, v, do, attention_bias=None, segment_ids=None, causal_block_size=None,
                             o=None, lse=None):
    """The sums of the backward's terms taken in absolute value, float64.

    Returns (mag_dq, mag_dk, mag_dv) [B,S,H,D]:

        mag_dq_i = scale sum_j |dS_ij| |k_j|,   mag_dk_j = scale sum_i |dS_ij| |q_i|,
        mag_dv_j = sum_i P_ij |dO_i|            (|.| element-wise on vectors)

    with P and dS the same quantities as in ``attention_backward``.  They are
    not part of the method: they bound how far a backward may move when its
    product operands dS and P are rounded, element by element, with relative
    error at most u before the sums (each term moves by at most u times its
    magnitude), which is how the tests hold a bf16 tensor-core backward to the
    exact gradients.  ``o`` / ``lse`` as in ``attention_backward``.
    """
    q = np.asarray(q)
    B, S, H, D = q.shape
    scale = 1.0 / math.sqrt(D)
    if o is None or lse is None:
        o, lse = attention_forward(q, k, v, attention_bias, segment_ids, causal_block_size)
    mq = np.zeros((B, S, H, D), dtype=np.float64)
    mk = np.zeros((B, S, H, D), dtype=np.float64)
    mv = np.zeros((B, S, H, D), dtype=np.float64)
    for b in range(B):
        seg_b = None if segment_ids is None else np.asarray(segment_ids)[b]
        bias_b = None if attention_bias is None else _f64(attention_bias)[b]
        for h in range(H):
            qh, kh, vh, doh = _f64(q[b, :, h]), _f64(k[b, :, h]), _f64(v[b, :, h]), _f64(do[b, :, h])
            oh, lse_h = _f64(o[b, :, h]), _f64(lse[b, h])
            for a, e in _row_chunks(S, S):
                rows = np.arange(a, e)
                vis = visible_mask(rows, S, causal_block_size, seg_b, bias_b)
                s = scale * (qh[a:e] @ kh.T)
                if bias_b is not None:
                    s = s + np.where(np.isfinite(bias_b), bias_b, 0.0)[None, :]
                has = np.isfinite(lse_h[a:e])
                P = np.where(vis & has[:, None], np.exp(s - np.where(has, lse_h[a:e], 0.0)[:, None]), 0.0)
                Dl = np.sum(doh[a:e] * oh[a:e], axis=1)
                dS = np.abs(P * (doh[a:e] @ vh.T - Dl[:, None]))
                mq[b, a:e, h] = scale * (dS @ np.abs(kh))
                mk[b, :, h] += scale * (dS.T @ np.abs(qh[a:e]))
                mv[b, :, h] += P.T @ np.abs(doh[a:e])
    return mq, mk, mv


def visible_count_rows(rows, S, causal_block_size=None, seg_b=None, bias_b=None):
    """Exact integer number of visible keys for each query row of one batch."""
    rows = np.asarray(rows, dtype=np.int64)
    out = np.zeros(len(rows), dtype=np.int64)
    for a, e in _row_chunks(len(rows), S):
        out[a:e] = visible_mask(rows[a:e], S, causal_block_size, seg_b, bias_b).sum(axis=1)
    return out


def visible_count_cols(S, causal_block_size=None, seg_b=None, bias_b=None):
    """Exact integer number of visible query rows for each key j of one batch.

    The column sums of the same mask as ``visible_count_rows`` (which keys
    take part follows "RingAttention核心功能全解析", 核心API调用: causal_block_size,
    segment_ids, attention_bias).
    """
    out = np.zeros(S, dtype=np.int64)
    rows = np.arange(S, dtype=np.int64)
    for a, e in _row_chunks(S, S):
        out += visible_mask(rows[a:e], S, causal_block_size, seg_b, bias_b).sum(axis=0)
    return out


def visible_pairs_total(B, H, S, causal_block_size=None, segment_ids=None, attention_bias=None):
    """Exact integer count of visible (i, j) pairs summed over all (b, h).

    Counted from the integer mask, one batch row at a time (heads share the
    mask).  This is the N_vis of the algorithmic FLOP count 4*D*N_vis.
    """
    total = 0
    for b in range(B):
        seg_b = None if segment_ids is None else np.asarray(segment_ids)[b]
        bias_b = None if attention_bias is None else np.asarray(attention_bias, dtype=np.float64)[b]
        total += int(visible_count_rows(np.arange(S), S, causal_block_size, seg_b, bias_b).sum())
    return total * H
