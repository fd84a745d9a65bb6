"""The 'boundary window' scheme that one page sketches, as a negative control.

The page "Ring Attention技术解析" (§2.2 pseudocode, §3.2 "重叠窗口") describes
each device computing attention of its own queries against its own block, and
only the last ``overlap`` queries of the block against the previous block's
keys and values, then concatenating.  That is not full attention: most
queries never see earlier blocks.  This helper reproduces that scheme (CPU,
float64) so a test can show the parity checker rejects a non-exact method.
"""

from __future__ import annotations

import math

import numpy as np


def _attend(q, k, v, qpos, kpos):
    D = q.shape[1]
    s = (q @ k.T) / math.sqrt(D)
    s = np.where(qpos[:, None] >= kpos[None, :], s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    return (e @ v) / e.sum(axis=1, keepdims=True)


def boundary_window_attention(q, k, v, ring_size, overlap):
    """Causal 'local block + boundary window' approximation, [B,S,H,D] float64."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, S, H, D = q.shape
    blk = S // ring_size
    out = np.zeros_like(q)
    for b in range(B):
        for h in range(H):
            for r in range(ring_size):
                a, e = r * blk, (r + 1) * blk
                pos = np.arange(a, e)
                local = _attend(q[b, a:e, h], k[b, a:e, h], v[b, a:e, h], pos, pos)
                if r > 0:
                    # the last `overlap` queries see the previous block's keys plus their own
                    tail = pos[-overlap:]
                    kp = np.arange(a - blk, e)
                    local[-overlap:] = _attend(q[b, tail, h], k[b, kp, h], v[b, kp, h], tail, kp)
                out[b, a:e, h] = local
    return out
