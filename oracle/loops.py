"""Pure-Python loops for the attention definition, tiny inputs only.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

An independent restatement of the definition in ``oracle.attention`` (same
page citations): every score, exponential and sum is a scalar Python float
operation with ``math.exp``; no numpy arithmetic is used.  Tests compare the
vectorised oracle against these loops on inputs of a few dozen tokens, so a
transposed operand, a wrong mask index or a dropped term in either one shows.
"""

from __future__ import annotations

import math


def _visible(i, j, c, seg, bias):
    if c and (i // c) < (j // c):
        return False
    if seg is not None and seg[i] != seg[j]:
        return False
    if bias is not None and bias[j] == -math.inf:
        return False
    return True


def forward_loops(q, k, v, bias=None, seg=None, c=None):
    """q, k, v: nested lists [S][D] of one (b, h); bias, seg: lists [S] or None.

    Returns (o [S][D], lse [S]) as Python floats.
    """
    S = len(q)
    D = len(q[0])
    scale = 1.0 / math.sqrt(D)
    o, lse = [], []
    for i in range(S):
        scores = []
        for j in range(S):
            if _visible(i, j, c, seg, bias):
                dot = 0.0
                for d in range(D):
                    dot += float(q[i][d]) * float(k[j][d])
                sc = scale * dot + (0.0 if bias is None else float(bias[j]))
                scores.append((j, sc))
        if not scores:
            o.append([0.0] * D)
            lse.append(-math.inf)
            continue
        m = max(sc for _, sc in scores)
        z = sum(math.exp(sc - m) for _, sc in scores)
        row = [0.0] * D
        for j, sc in scores:
            w = math.exp(sc - m) / z
            for d in range(D):
                row[d] += w * float(v[j][d])
        o.append(row)
        lse.append(m + math.log(z))
    return o, lse


def backward_loops(q, k, v, do, bias=None, seg=None, c=None):
    """Gradients (dq, dk, dv), each [S][D], of L = sum_i <dO_i, o_i> for one (b, h)."""
    S = len(q)
    D = len(q[0])
    scale = 1.0 / math.sqrt(D)
    o, lse = forward_loops(q, k, v, bias, seg, c)
    dq = [[0.0] * D for _ in range(S)]
    dk = [[0.0] * D for _ in range(S)]
    dv = [[0.0] * D for _ in range(S)]
    for i in range(S):
        if lse[i] == -math.inf:
            continue
        dl = sum(float(do[i][d]) * o[i][d] for d in range(D))
        for j in range(S):
            if not _visible(i, j, c, seg, bias):
                continue
            dot = sum(float(q[i][d]) * float(k[j][d]) for d in range(D))
            s = scale * dot + (0.0 if bias is None else float(bias[j]))
            p = math.exp(s - lse[i])
            dp = sum(float(do[i][d]) * float(v[j][d]) for d in range(D))
            ds = p * (dp - dl)
            for d in range(D):
                dq[i][d] += scale * ds * float(k[j][d])
                dk[j][d] += scale * ds * float(q[i][d])
                dv[j][d] += p * float(do[i][d])
    return dq, dk, dv
