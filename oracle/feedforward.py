"""The blockwise feed-forward network, float64 (the oracle).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

What it computes.  The pages export ``blockwise_feedforward`` next to
``ringattention`` ([RA-core] 核心API调用: ``from ringattention import
ringattention, blockwise_feedforward``) and name the model configuration
they shard, ``LLaMAConfig`` ([RA-core] 核心技术原理 3).  They print no formula.
The plainest reading (listed in the design notes): the position-wise
feed-forward network of that model, a SwiGLU without biases,

    h_t = silu(x_t W1^T) * (x_t W3^T)          silu(a) = a / (1 + exp(-a))
    y_t = h_t W2^T

for every token t, evaluated over the sequence one chunk of ``chunk_size``
tokens at a time (the "blockwise" part: only a chunk's intermediate h is
held at once, so memory stays linear in the sequence length, as for the
attention).  Chunking does not change the result; rows are independent.

Shapes: x [T, d_model]; W1, W3 [d_ff, d_model]; W2 [d_model, d_ff] (each
weight stored output-major, like a linear layer's weight); y [T, d_model].
"""

from __future__ import annotations

import numpy as np


def silu(a):
    """a * sigmoid(a), written out: a / (1 + exp(-a)), stable for large |a|."""
    a = np.asarray(a, dtype=np.float64)
    out = np.empty_like(a)
    pos = a >= 0
    out[pos] = a[pos] / (1.0 + np.exp(-a[pos]))
    e = np.exp(a[~pos])
    out[~pos] = a[~pos] * e / (1.0 + e)
    return out


def blockwise_feedforward(x, w1, w3, w2, chunk_size=None, return_hidden=False):
    """y = (silu(x W1^T) * (x W3^T)) W2^T, chunk by chunk.  float64.

    ``return_hidden``: also return h [T, d_ff] (the gated hidden layer)."""
    x = np.asarray(x, dtype=np.float64)
    w1, w3, w2 = (np.asarray(w, dtype=np.float64) for w in (w1, w3, w2))
    T = x.shape[0]
    c = T if not chunk_size else int(chunk_size)
    y = np.zeros((T, w2.shape[0]), dtype=np.float64)
    h_all = np.zeros((T, w1.shape[0]), dtype=np.float64) if return_hidden else None
    for a in range(0, T, max(c, 1)):
        xc = x[a:a + c]
        h = silu(xc @ w1.T) * (xc @ w3.T)
        y[a:a + c] = h @ w2.T
        if return_hidden:
            h_all[a:a + c] = h
    return (y, h_all) if return_hidden else y
