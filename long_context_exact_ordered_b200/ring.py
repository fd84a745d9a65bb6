"""Ring attention across the ranks of a process group: the sequence sharded over GPUs.

The pages' system ("Ring Attention技术解析" §2.2 and §4.2; "手把手拆解RingAttention"
§2; "RingAttention核心功能全解析" 核心技术原理 2 and 3): every device keeps its
block of queries; the key/value blocks travel round a ring of devices, each
device sending its current block to the next device and receiving the
previous device's, while it computes attention of its queries against the
block it holds.  After G steps every query has met every key, and the
running online-softmax state gives exact attention.

Here one process drives one GPU.  Per step the rank

* posts the exchange of the block it holds (keys, values and, when given,
  their segment ids and bias) on a communication stream: send to rank+1,
  receive from rank-1, into the other half of a local double buffer
  (``torch.distributed`` P2P: NCCL between GPUs, gloo between CPU
  processes);
* runs ``ra_step`` (the tensor-core forward kernel in ring-step mode) for its
  query chunks against the chunks of the block it holds, on the compute
  stream, merging into per-chunk fp32 running states;
* makes the compute stream wait for the exchange before the next step.

Causal load balance (the pages are silent on it; this is the usual zig-zag
split): with ``layout="zigzag"`` the sequence is cut into 2G chunks and rank
r holds chunks r and 2G-1-r, so every rank has the same number of visible
(query, key) pairs under causal masking.  ``layout="contiguous"`` gives rank
r the r-th of G blocks, as in the pages' figure.  Masks use global token
positions, so the layout never changes the result.

Blocks that causal masking hides entirely from a query chunk are skipped on
the host.  The module moves tensors and orders launches; every arithmetic
step runs in the library's kernels (``ra_step``, ``ra_finalize``).
"""

from __future__ import annotations

import torch
import torch.distributed as dist

from . import api


def chunk_layout(rank: int, world: int, s_local: int, layout: str = "zigzag"):
    """This rank's tokens as [(local_start, global_start, length)].

    ``s_local`` tokens per rank; "contiguous": global block ``rank``;
    "zigzag": chunks ``rank`` and ``2*world-1-rank`` of 2*world chunks of
    ``s_local // 2`` tokens (``s_local`` must be even)."""
    if layout == "contiguous":
        return [(0, rank * s_local, s_local)]
    if layout == "zigzag":
        if s_local % 2:
            raise ValueError("zigzag layout needs an even number of tokens per rank")
        half = s_local // 2
        return [(0, rank * half, half), (half, (2 * world - 1 - rank) * half, half)]
    raise ValueError(f"unknown layout {layout!r}")


def shard(x: torch.Tensor, rank: int, world: int, layout: str = "zigzag", dim: int = 1) -> torch.Tensor:
    """This rank's part of a full-sequence tensor (sequence along ``dim``), in
    the order ``chunk_layout`` gives."""
    S = x.shape[dim]
    if S % world:
        raise ValueError("sequence length must be a multiple of the world size")
    parts = [x.narrow(dim, g, n) for _, g, n in chunk_layout(rank, world, S // world, layout)]
    return torch.cat(parts, dim).contiguous()


def unshard(parts, world: int, layout: str = "zigzag", dim: int = 1) -> torch.Tensor:
    """Inverse of ``shard``: the full-sequence tensor from every rank's part."""
    s_local = parts[0].shape[dim]
    pieces = []
    for r, p in enumerate(parts):
        for l0, g0, n in chunk_layout(r, world, s_local, layout):
            pieces.append((g0, p.narrow(dim, l0, n)))
    pieces.sort(key=lambda x: x[0])
    return torch.cat([p for _, p in pieces], dim)


def _hidden(q_start, q_len, k_start, causal_block_size):
    """Whether causal masking hides every key from k_start on from the queries [q_start, q_start + q_len)."""
    if not causal_block_size:
        return False
    c = int(causal_block_size)
    return k_start // c > (q_start + q_len - 1) // c


def _segment_ranges(segment_ids, chunks):
    """Per chunk of this rank ((local start, global start, length) triples),
    the smallest and largest segment id of every batch row: int64 [chunks, B, 2].
    An empty chunk gets a range that meets no other."""
    B = segment_ids.shape[0]
    out = torch.empty((len(chunks), B, 2), dtype=torch.int64, device=segment_ids.device)
    for i, (ql, _, qn) in enumerate(chunks):
        if qn == 0:
            out[i, :, 0], out[i, :, 1] = 1 << 62, -(1 << 62)
            continue
        part = segment_ids[:, ql:ql + qn]
        out[i, :, 0] = part.amin(dim=1)
        out[i, :, 1] = part.amax(dim=1)
    return out


def _segments_disjoint(q_range, k_range):
    """Whether no batch row has a key segment id that also occurs among its
    queries, judged by their ranges ([B, 2] each): a step over such a pair of
    chunks would leave the running state unchanged."""
    return bool(((q_range[:, 1] < k_range[:, 0]) | (q_range[:, 0] > k_range[:, 1])).all())


class _Exchange:
    """The ring's double-buffered key/value exchange: send the held block to
    rank+1, receive the next one from rank-1."""

    def __init__(self, tensors, group, comm_stream):
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        # the caller's tensors are only read (step 0); the blocks that arrive
        # alternate between two buffers of this exchange's own
        self.own = list(tensors)
        self.bufs = [[torch.empty_like(t) for t in tensors] for _ in range(2)]
        self.cuda = tensors[0].is_cuda
        self.comm = comm_stream if (self.cuda and comm_stream is not None) else (
            torch.cuda.Stream(tensors[0].device) if self.cuda else None)
        self.pending = None

    def held(self, t):
        return self.own if t == 0 else self.bufs[t % 2]

    def start(self, t):
        """Post the exchange that brings step t+1's block into the other buffer."""
        send, recv = self.held(t), self.bufs[(t + 1) % 2]
        nxt, prv = (self.rank + 1) % self.world, (self.rank - 1) % self.world
        if self.group is not None:                    # P2P peers are global ranks
            nxt, prv = dist.get_global_rank(self.group, nxt), dist.get_global_rank(self.group, prv)
        ops = []
        for s, r in zip(send, recv):
            ops.append(dist.P2POp(dist.isend, s, nxt, self.group))
            ops.append(dist.P2POp(dist.irecv, r, prv, self.group))
        if self.cuda:
            # the receive buffer was read by the previous step's kernels, queued on the compute stream
            ready = torch.cuda.Event()
            ready.record(torch.cuda.current_stream())
            with torch.cuda.stream(self.comm):
                self.comm.wait_event(ready)
                self.pending = dist.batch_isend_irecv(ops)
        else:
            self.pending = dist.batch_isend_irecv(ops)

    def finish(self):
        """The compute stream (or the caller, on CPU) waits for the posted exchange."""
        if self.pending is not None:
            for w in self.pending:
                w.wait()
            self.pending = None


def ring_attention_forward(q, k, v, attention_bias=None, segment_ids=None, causal_block_size=1, group=None,
                           layout="zigzag", comm_stream=None, step=None, finalize=None):
    """Exact attention of this rank's queries over the whole sharded sequence.

    q, k, v: this rank's tokens [B, S_local, H, D] (``shard`` of the full
    tensors with the same ``layout``); attention_bias: fp32 [B, S_local] or
    None; segment_ids: int32 [B, S_local] or None (this rank's keys and
    queries).  Returns (o [B, S_local, H, D], lse fp32 [B, H, S_local]) for
    this rank's queries, in local order.  Every rank of ``group`` must call
    it with the same shapes, and all with segment ids or all without: with
    them, the ranks first all-gather their chunks' segment ranges.  ``step`` / ``finalize`` default to the
    library's ``ring_step`` / ``finalize``; the CPU tests pass the oracle's
    here to check the exchange protocol without a GPU.
    """
    step = api.ring_step if step is None else step
    finalize = api.finalize if finalize is None else finalize
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    B, s_local, H, D = q.shape
    chunks = chunk_layout(rank, world, s_local, layout)
    states = [api.init_state(B, n, H, D, q.device) for _, _, n in chunks]
    held = [x.contiguous() for x in [k, v] + ([attention_bias] if attention_bias is not None else []) + (
        [segment_ids] if segment_ids is not None else [])]
    ex = _Exchange(held, group, comm_stream) if world > 1 else None
    # With segment ids, every rank learns every chunk's segment range once (one
    # all-gather of a few integers), so that steps over a (query chunk, key
    # chunk) pair with disjoint segments are skipped on the host, like the
    # pairs causal masking hides.
    seg_ranges = None
    if segment_ids is not None:
        mine_r = _segment_ranges(segment_ids, chunks)
        if world > 1:
            parts = [torch.empty_like(mine_r) for _ in range(world)]
            dist.all_gather(parts, mine_r, group=group)
            seg_ranges = [x.cpu() for x in parts]
        else:
            seg_ranges = [mine_r.cpu()]
    for t in range(world):
        cur = ex.held(t) if ex else held
        if ex and t < world - 1:
            ex.start(t)
        src = (rank - t) % world                      # the block that started t ranks behind
        kc, vc = cur[0], cur[1]
        bias_c = cur[2] if attention_bias is not None else None
        seg_c = cur[-1] if segment_ids is not None else None
        for qi, ((ql, qg, qn), (acc, m, l)) in enumerate(zip(chunks, states)):
            seg_q = None if segment_ids is None else segment_ids[:, ql:ql + qn].contiguous()
            for ki, (kl, kg, kn) in enumerate(chunk_layout(src, world, s_local, layout)):
                if _hidden(qg, qn, kg, causal_block_size):
                    continue
                if seg_ranges is not None and _segments_disjoint(seg_ranges[rank][qi], seg_ranges[src][ki]):
                    continue
                step(q[:, ql:ql + qn], kc[:, kl:kl + kn], vc[:, kl:kl + kn], qg, kg, acc, m, l,
                     bias_blk=None if bias_c is None else bias_c[:, kl:kl + kn].contiguous(),
                     seg_q=seg_q, seg_k=None if seg_c is None else seg_c[:, kl:kl + kn].contiguous(),
                     causal_block_size=causal_block_size)
        if ex:
            ex.finish()
    o = torch.empty_like(q)
    lse = torch.empty((B, H, s_local), dtype=torch.float32, device=q.device)
    for (ql, qg, qn), (acc, m, l) in zip(chunks, states):
        finalize(acc, m, l, q.dtype, out=o[:, ql:ql + qn], lse=lse[:, :, ql:ql + qn])
    return o, lse

