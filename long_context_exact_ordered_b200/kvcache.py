"""Ring steps against a growing key/value cache: the serving side of the ring.

Page "Ring Attention技术解析" §7 (推理优化): at inference the keys and values of
the tokens already processed are kept, new tokens attend to them, and
requests that begin with the same prefix share that prefix's cache.  Here a
cache holds the keys and values of its tokens on the device; a chunk of new
queries attends to the cache block by block with one ``ra_step`` per block
(the ring's step loop, the cache's blocks playing the visiting blocks),
merging into one fp32 running state, then ``ra_finalize``.  Prefill chunks
and single-token decode steps are the same call.

Prefix sharing: a cache of batch 1 can be the ``prefix`` of a cache of batch
B (B requests continuing the same prefix).  Every request's queries then
read the one prefix copy (``ra_step`` accepts a key/value block of batch 1
for a query block of batch B), and only the continuations are stored per
request.  Positions are global: a cache's tokens follow its prefix's.

This module only allocates the cache buffers and orders the calls; every
arithmetic step runs in the library's kernels.
"""

from __future__ import annotations

import torch

from . import api


class KVCache:
    """Keys and values of a growing sequence, [batch, capacity, heads, head_dim].

    ``block``: tokens per ``ra_step`` call when attending (a multiple of 128
    keeps every call on whole key tiles).  ``prefix``: an optional cache of
    batch 1 whose tokens come first and are shared by every batch row of
    this cache.
    """

    def __init__(self, batch, heads, head_dim, capacity, block=4096, dtype=torch.bfloat16, device=None,
                 prefix: "KVCache | None" = None):
        if prefix is not None and prefix.batch != 1 and prefix.batch != batch:
            raise ValueError("a prefix cache must have batch 1 (shared) or this cache's batch")
        if prefix is not None and (prefix.heads, prefix.head_dim, prefix.dtype) != (heads, head_dim, dtype):
            raise ValueError("prefix cache has a different head layout or dtype")
        device = torch.device("cuda") if device is None else torch.device(device)
        self.batch, self.heads, self.head_dim, self.dtype = batch, heads, head_dim, dtype
        self.capacity, self.block, self.prefix = capacity, int(block), prefix
        self.k = torch.empty((batch, capacity, heads, head_dim), dtype=dtype, device=device)
        self.v = torch.empty_like(self.k)
        self.length = 0

    @property
    def offset(self) -> int:
        """Global position of this cache's first token (the prefix's length)."""
        return 0 if self.prefix is None else self.prefix.total_length

    @property
    def total_length(self) -> int:
        return self.offset + self.length

    def append(self, k, v):
        """Store the keys / values [batch, n, heads, head_dim] of the next n tokens."""
        n = k.shape[1]
        if self.length + n > self.capacity:
            raise ValueError("KV cache capacity exceeded")
        self.k[:, self.length:self.length + n].copy_(k)
        self.v[:, self.length:self.length + n].copy_(v)
        self.length += n

    def chain(self):
        """The caches whose tokens this cache's queries see, first token first."""
        out, c = [], self
        while c is not None:
            out.append(c)
            c = c.prefix
        return out[::-1]

    def attend(self, q, q_off=None, causal_block_size=1, step=None, finalize=None):
        """Attention of queries q [batch, n, heads, head_dim] at global positions
        q_off .. q_off+n-1 (default: the last n cached positions) over every
        cached key, including the prefix's.  Returns (o, lse).  ``step`` /
        ``finalize`` default to the library's ``ring_step`` / ``finalize``."""
        step = api.ring_step if step is None else step
        finalize = api.finalize if finalize is None else finalize
        B, n, H, D = q.shape
        if B != self.batch:
            raise ValueError("query batch must equal the cache's batch")
        if q_off is None:
            q_off = self.total_length - n
        acc, m, l = api.init_state(B, n, H, D, q.device)
        q_last = q_off + n - 1
        for c in self.chain():
            for s in range(0, c.length, self.block):
                e = min(c.length, s + self.block)
                k_off = c.offset + s
                if causal_block_size and k_off // causal_block_size > q_last // causal_block_size:
                    break                      # this block and every later one lie after the queries
                step(q, c.k[:, s:e], c.v[:, s:e], q_off, k_off, acc, m, l, causal_block_size=causal_block_size)
        return finalize(acc, m, l, q.dtype)
