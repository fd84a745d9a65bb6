"""The cross-rank ring (long_context_exact_ordered_b200.ring) on CPU processes.

World sizes 2, 3 and 4 over gloo: every rank holds its shard of the sequence,
key/value blocks (with their segment ids and bias) travel round the ring
through torch.distributed point-to-point exchanges, and the per-step
arithmetic is the oracle's online-softmax step in float64 (passed in as the
step function, since these processes have no GPU).  Every rank's output must
equal the float64 definition of full attention on its own tokens, for both
the zig-zag and the contiguous layouts.  On GPUs the same exchange code runs
over NCCL with ra_step on the tensor cores.
"""

from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from long_context_exact_ordered_b200 import ring
from oracle_steps import oracle_finalize as _oracle_finalize
from oracle_steps import oracle_step as _oracle_step


def _inputs(S, seed, segments, bias):
    g = torch.Generator().manual_seed(seed)
    B, H, D = 2, 2, 16
    q, k, v = (torch.randn((B, S, H, D), generator=g, dtype=torch.float64) for _ in range(3))
    seg = None
    if segments:
        lengths = [5, 17, 3, 40, S]
        ids, n = [], 0
        for i, L in enumerate(lengths):
            L = min(L, S - n)
            ids += [i] * L
            n += L
            if n == S:
                break
        seg = torch.tensor(ids, dtype=torch.int32).unsqueeze(0).expand(B, S).contiguous()
    bb = None
    if bias:
        bb = torch.randn((B, S), generator=g, dtype=torch.float64)
        bb[:, torch.randint(0, S, (S // 6,), generator=g)] = float("-inf")
    return q, k, v, seg, bb


def _worker(rank, world, port, cases, errors):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        for layout, c, segments, bias in cases:
            S = 24 * world
            q, k, v, seg, bb = _inputs(S, 7 + world, segments, bias)
            ro, rl = oracle.attention_forward(q.numpy(), k.numpy(), v.numpy(), None if bb is None else bb.numpy(),
                                              None if seg is None else seg.numpy(), c)
            sh = lambda x: None if x is None else ring.shard(x, rank, world, layout)
            mine = [sh(x) for x in (q, k, v, bb, seg)]
            kept = [None if x is None else x.clone() for x in mine]
            calls = []

            def counted_step(*a, **kw):
                calls.append(1)
                return _oracle_step(*a, **kw)

            o, lse = ring.ring_attention_forward(*mine, causal_block_size=c, layout=layout, step=counted_step,
                                                 finalize=_oracle_finalize)
            if segments:
                # the same ring without segment ids makes every step the mask allows
                plain = []
                ring.ring_attention_forward(*mine[:4], None, causal_block_size=c, layout=layout,
                                            step=lambda *a, **kw: (plain.append(1), _oracle_step(*a, **kw))[1],
                                            finalize=_oracle_finalize)
                if not len(calls) < len(plain):
                    errors.put(f"rank {rank} {layout}: no step skipped for disjoint segments "
                               f"({len(calls)} vs {len(plain)})")
            if any(a is not None and not torch.equal(a, b) for a, b in zip(mine, kept)):
                errors.put(f"rank {rank} {layout}: the caller's tensors were modified")
            want_o = ring.shard(torch.from_numpy(ro), rank, world, layout)
            want_l = ring.shard(torch.from_numpy(rl), rank, world, layout, dim=2)
            err = float((o - want_o).abs().max())
            fin = torch.isfinite(want_l)
            lerr = float((lse.double()[fin] - want_l[fin]).abs().max()) if fin.any() else 0.0
            pattern = bool(torch.equal(torch.isfinite(lse), fin))
            if not (err <= 1e-6 and lerr <= 1e-5 and pattern):
                errors.put(f"rank {rank} {layout} c={c} seg={segments} bias={bias}: o {err:.2e} lse {lerr:.2e}")
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


CASES = [("zigzag", 1, False, False), ("contiguous", 1, False, False), ("zigzag", None, True, True),
         ("zigzag", 3, True, False), ("contiguous", 1, False, True)]


@pytest.mark.parametrize("world", [2, 3, 4])
def test_ring_across_ranks_equals_full_attention(world):
    ctx = mp.get_context("spawn")
    errors = ctx.SimpleQueue()
    mp.start_processes(_worker, args=(world, _free_port(), CASES, errors), nprocs=world, join=True,
                       start_method="spawn")
    found = []
    while not errors.empty():
        found.append(errors.get())
    assert not found, "\n".join(found)


def test_layouts_round_trip_and_balance():
    world, S = 4, 64
    x = torch.arange(S).view(1, S, 1, 1).float()
    for layout in ("zigzag", "contiguous"):
        parts = [ring.shard(x, r, world, layout) for r in range(world)]
        assert torch.equal(ring.unshard(parts, world, layout), x)
    # zig-zag gives every rank the same number of causal (query, key) pairs
    pairs = []
    for r in range(world):
        pos = ring.shard(x, r, world, "zigzag").view(-1).long()
        pairs.append(int((pos + 1).sum()))
    assert len(set(pairs)) == 1
    contiguous = [int((ring.shard(x, r, world, "contiguous").view(-1).long() + 1).sum()) for r in range(world)]
    assert len(set(contiguous)) == world


def test_hidden_blocks():
    assert ring._hidden(0, 16, 16, 1) and not ring._hidden(0, 16, 15, 1)
    assert not ring._hidden(0, 16, 16, None)
    assert not ring._hidden(0, 16, 17, 6) and ring._hidden(0, 16, 18, 6)
