"""Ring-blockwise route to the same attention, float64 (oracle self-checks).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

This follows the method's own steps rather than the plain definition, so
that the oracle's self-tests can show the two routes agree:

1. The sequence is cut into P contiguous ring blocks ([RA-tech] §2.2,
   "序列分块"); virtual rank r holds query block r and, at first, key/value
   block r.
2. At every step each rank sends its current key/value block to the next
   rank and receives one from the previous rank ([RA-tech] §2.2 pseudocode,
   send to ``next_rank``, receive from ``prev_rank``; [RA-LWM] §1: queries
   stay, keys and values travel).  So at step t rank r holds block
   (r - t) mod P.  ``order`` permutes the steps for invariance tests.
3. Inside a step the local queries and the visiting keys are processed in
   chunks of ``query_chunk_size`` x ``key_chunk_size`` ([RA-core] 核心技术原理
   1, ``blockwise_kwargs``).
4. The partial results are combined exactly.  The pages only state that the
   result is complete global attention ([RA-LWM] §1); the combination used
   here is the standard online softmax (running max m, running sum l, output
   accumulator rescaled by exp(m_old - m_new)) and, for already-normalised
   partials, the log-sum-exp merge.  Which of the two is used does not change
   the result.
"""

from __future__ import annotations

import math

import numpy as np

from .attention import causal_ok


def online_step(state, q_c, k_c, v_c, qpos, kpos, causal_block_size=None,
                seg_q=None, seg_k=None, bias_k=None):
    """One online-softmax update of ``state`` = (m, l, acc) with a key chunk.

    q_c [n, D], k_c / v_c [m, D] float64; qpos / kpos global token indices;
    seg_q [n], seg_k [m], bias_k [m] or None.  m, l [n]; acc [n, D].  m and
    the scores are in natural-log units.  Returns the new state.
    """
    m, l, acc = state
    D = q_c.shape[1]
    scale = 1.0 / math.sqrt(D)
    vis = causal_ok(np.asarray(qpos)[:, None], np.asarray(kpos)[None, :], causal_block_size)
    if seg_q is not None:
        vis = vis & (np.asarray(seg_q)[:, None] == np.asarray(seg_k)[None, :])
    s = scale * (q_c @ k_c.T)
    if bias_k is not None:
        bias_k = np.asarray(bias_k, dtype=np.float64)
        vis = vis & (bias_k[None, :] > -np.inf)
        s = s + np.where(np.isfinite(bias_k), bias_k, 0.0)[None, :]
    s = np.where(vis, s, -np.inf)
    m_new = np.maximum(m, s.max(axis=1))
    live = np.isfinite(m_new)
    ref = np.where(live, m_new, 0.0)
    alpha = np.where(np.isfinite(m), np.exp(np.where(np.isfinite(m), m, 0.0) - ref), 0.0)
    p = np.where(vis, np.exp(s - ref[:, None]), 0.0)
    l_new = alpha * l + p.sum(axis=1)
    acc_new = alpha[:, None] * acc + p @ v_c
    return m_new, l_new, acc_new


def finalize(state):
    """(m, l, acc) -> (o, lse); rows with l == 0 give o = 0 and lse = -inf."""
    m, l, acc = state
    has = l > 0
    o = np.where(has[:, None], acc / np.where(has, l, 1.0)[:, None], 0.0)
    lse = np.where(has, m + np.log(np.where(has, l, 1.0)), -np.inf)
    return o, lse


def lse_merge(o_a, lse_a, o_b, lse_b):
    """Merge two normalised partial attentions over disjoint key sets.

    lse = log(exp(lse_a) + exp(lse_b)) = max + log1p(exp(-|lse_a - lse_b|));
    o   = o_a exp(lse_a - lse) + o_b exp(lse_b - lse).
    Rows where both sides are empty stay empty (o = 0, lse = -inf).
    """
    lse_a = np.asarray(lse_a, dtype=np.float64)
    lse_b = np.asarray(lse_b, dtype=np.float64)
    hi = np.maximum(lse_a, lse_b)
    lo = np.minimum(lse_a, lse_b)
    live = np.isfinite(hi)
    both = live & np.isfinite(lo)
    gap = np.where(both, np.where(both, lo, 0.0) - np.where(both, hi, 0.0), -np.inf)
    lse = np.where(live, np.where(live, hi, 0.0) + np.log1p(np.exp(gap)), -np.inf)
    ref = np.where(live, lse, 0.0)
    wa = np.where(np.isfinite(lse_a), np.exp(np.where(np.isfinite(lse_a), lse_a, 0.0) - ref), 0.0)
    wb = np.where(np.isfinite(lse_b), np.exp(np.where(np.isfinite(lse_b), lse_b, 0.0) - ref), 0.0)
    o = wa[..., None] * np.asarray(o_a, dtype=np.float64) + wb[..., None] * np.asarray(o_b, dtype=np.float64)
    return o, lse


def ring_blockwise_reference(q, k, v, attention_bias=None, segment_ids=None, causal_block_size=None,
                             ring_size=1, query_chunk_size=None, key_chunk_size=None,
                             order=None, merge="online"):
    """Ring attention over P = ``ring_size`` virtual ranks.

    ``merge="online"`` carries one running (m, l, acc) per query row across
    all steps; ``merge="lse"`` finalizes each step's partial separately and
    combines the partials with ``lse_merge``.  ``order`` is a permutation of
    range(P) giving the step offsets t (default 0, 1, ..., P-1).

    Returns o [B,S,H,D], lse [B,H,S] float64.
    """
    q = np.asarray(q)
    B, S, H, D = q.shape
    P = int(ring_size)
    if S % P:
        raise ValueError("sequence length must be a multiple of ring_size")
    blk = S // P
    qc = blk if query_chunk_size is None else int(query_chunk_size)
    kc = blk if key_chunk_size is None else int(key_chunk_size)
    if blk % qc or blk % kc:
        raise ValueError("chunk sizes must divide the ring block")
    steps = list(range(P)) if order is None else [int(t) for t in order]
    if sorted(steps) != list(range(P)):
        raise ValueError("order must be a permutation of range(ring_size)")
    o = np.zeros((B, S, H, D), dtype=np.float64)
    lse = np.full((B, H, S), -np.inf, dtype=np.float64)
    for b in range(B):
        seg_b = None if segment_ids is None else np.asarray(segment_ids)[b]
        bias_b = None if attention_bias is None else np.asarray(attention_bias, dtype=np.float64)[b]
        for h in range(H):
            qh = np.asarray(q[b, :, h], dtype=np.float64)
            kh = np.asarray(k[b, :, h], dtype=np.float64)
            vh = np.asarray(v[b, :, h], dtype=np.float64)
            for r in range(P):                      # virtual rank r: query block r
                for qa in range(r * blk, (r + 1) * blk, qc):
                    qpos = np.arange(qa, qa + qc)
                    n = len(qpos)
                    running = (np.full(n, -np.inf), np.zeros(n), np.zeros((n, D)))
                    merged = (np.zeros((n, D)), np.full(n, -np.inf))
                    for t in steps:                 # step t: KV block (r - t) mod P
                        src = (r - t) % P
                        part = (np.full(n, -np.inf), np.zeros(n), np.zeros((n, D)))
                        for ka in range(src * blk, (src + 1) * blk, kc):
                            kpos = np.arange(ka, ka + kc)
                            args = (qh[qpos], kh[kpos], vh[kpos], qpos, kpos, causal_block_size,
                                    None if seg_b is None else seg_b[qpos],
                                    None if seg_b is None else seg_b[kpos],
                                    None if bias_b is None else bias_b[kpos])
                            if merge == "online":
                                running = online_step(running, *args)
                            else:
                                part = online_step(part, *args)
                        if merge != "online":
                            po, pl = finalize(part)
                            merged = lse_merge(merged[0], merged[1], po, pl)
                    ob, lb = finalize(running) if merge == "online" else merged
                    o[b, qpos, h] = ob
                    lse[b, h, qpos] = lb
    return o, lse
