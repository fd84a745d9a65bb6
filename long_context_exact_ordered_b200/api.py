"""Python binding of the C ABI: argument marshalling only.

Every computation runs in the CUDA kernels of ``libringattn.so``.  torch
provides device memory (outputs and workspace are ``torch.empty``), the
current CUDA stream, and nothing else.  Names follow the pages' API
("RingAttention核心功能全解析" 核心API调用: ``ringattention(xq, xk, xv,
attention_bias, segment_ids, blockwise_kwargs)``).
"""

from __future__ import annotations

import contextlib
import ctypes

import torch

from . import _lib
from ._lib import RA_BF16, RA_F32, RA_I32, RA_MAX_RING, RaHostStep, RaParams, RaTensor, check, load

_DT = {torch.float32: RA_F32, torch.bfloat16: RA_BF16, torch.int32: RA_I32}


def _tensor(t: torch.Tensor | None):
    if t is None:
        return None
    if t.dtype not in _DT:
        raise TypeError(f"unsupported dtype {t.dtype}")
    r = RaTensor()
    r.data = t.data_ptr() if t.numel() else 0
    r.dtype = _DT[t.dtype]
    r.ndim = t.dim()
    for i in range(t.dim()):
        r.shape[i] = t.shape[i]
        r.stride[i] = t.stride(i)
    return r


def _ref(x):
    return None if x is None else ctypes.byref(x)


def _params(S: int, query_chunk_size, key_chunk_size, causal_block_size, ring_size, ring_order,
            prof_events=None) -> RaParams:
    p = RaParams()
    if prof_events is not None:
        for ev in prof_events:
            if not ev.cuda_event:      # torch creates the CUDA event lazily, on its first record
                ev.record()
        p.prof_event_begin = prof_events[0].cuda_event
        p.prof_event_end = prof_events[1].cuda_event
    blk = max(1, S // max(1, ring_size))
    p.query_chunk_size = blk if query_chunk_size is None else int(query_chunk_size)
    p.key_chunk_size = blk if key_chunk_size is None else int(key_chunk_size)
    p.causal_block_size = 0 if not causal_block_size else int(causal_block_size)
    p.ring_size = int(ring_size)
    if ring_order is not None:
        order = [int(x) for x in ring_order]
        if len(order) != ring_size or len(order) > RA_MAX_RING:
            raise ValueError("ring_order must have ring_size entries")
        for i, x in enumerate(order):
            p.ring_order[i] = x
        p.use_ring_order = 1
    return p


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def workspace_size(which: int, q: torch.Tensor, params: RaParams, has_bias: bool, has_segments: bool) -> int:
    n = load().ra_workspace_size(which, ctypes.byref(_tensor(q)), ctypes.byref(params), int(has_bias),
                                 int(has_segments))
    if n == ctypes.c_size_t(-1).value:
        raise ValueError("invalid arguments for ra_workspace_size")
    return n


def _workspace(nbytes: int, device) -> torch.Tensor | None:
    if nbytes == 0:
        return None
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def ringattention(q, k, v, attention_bias=None, segment_ids=None, query_chunk_size=512, key_chunk_size=512,
                  causal_block_size=None, ring_size=1, ring_order=None, out=None, lse=None, workspace=None,
                  prof_events=None):
    """Exact attention over ``ring_size`` virtual ring ranks.  Returns (o, lse).

    q, k, v: [B, S, H, D] bf16 (tensor-core path) or fp32 (CUDA-core path),
    head dim contiguous.  attention_bias: fp32 [B, S] or None (additive per
    key, -inf masks).  segment_ids: int32 [B, S] or None.
    causal_block_size: None/0 non-causal, c >= 1 block-causal.
    Chunk sizes must divide S / ring_size (they group the kernels' tiles and
    do not change the result); ``None`` means one chunk per ring block.
    ``prof_events``: optional (begin, end) torch.cuda.Event pair recorded
    around the main kernel only.
    """
    B, S, H, D = q.shape
    p = _params(S, query_chunk_size, key_chunk_size, causal_block_size, ring_size, ring_order, prof_events)
    if out is None:
        out = torch.empty_like(q, memory_format=torch.contiguous_format)
    if lse is None:
        lse = torch.empty((B, H, S), dtype=torch.float32, device=q.device)
    need = workspace_size(0, q, p, attention_bias is not None, segment_ids is not None)
    if workspace is None or workspace.numel() < need:
        workspace = _workspace(need, q.device)
    tq, tk, tv, to, tl = _tensor(q), _tensor(k), _tensor(v), _tensor(out), _tensor(lse)
    tb, ts = _tensor(attention_bias), _tensor(segment_ids)
    code = load().ra_forward(ctypes.byref(tq), ctypes.byref(tk), ctypes.byref(tv), _ref(tb), _ref(ts),
                             ctypes.byref(p), ctypes.byref(to), ctypes.byref(tl),
                             None if workspace is None else workspace.data_ptr(), need, _stream())
    check(code, "ra_forward")
    return out, lse


def ringattention_static(q, k, v, attention_bias=None, segment_ids=None, query_chunk_size=512,
                         key_chunk_size=512, causal_block_size=None, ring_size=1, ring_order=None, out=None,
                         lse=None):
    """ringattention without any device allocation by the library: its scratch is a
    fixed static device array (see ra_forward_static).  For callers that cannot
    allocate device memory; ``out`` and ``lse`` may be preallocated so that this
    wrapper allocates nothing either."""
    B, S, H, D = q.shape
    p = _params(S, query_chunk_size, key_chunk_size, causal_block_size, ring_size, ring_order)
    if out is None:
        out = torch.empty_like(q, memory_format=torch.contiguous_format)
    if lse is None:
        lse = torch.empty((B, H, S), dtype=torch.float32, device=q.device)
    tq, tk, tv, to, tl = _tensor(q), _tensor(k), _tensor(v), _tensor(out), _tensor(lse)
    tb, ts = _tensor(attention_bias), _tensor(segment_ids)
    code = load().ra_forward_static(ctypes.byref(tq), ctypes.byref(tk), ctypes.byref(tv), _ref(tb), _ref(ts),
                                    ctypes.byref(p), ctypes.byref(to), ctypes.byref(tl), _stream())
    check(code, "ra_forward_static")
    return out, lse


def ringattention_backward(q, k, v, o, lse, do, attention_bias=None, segment_ids=None, query_chunk_size=512,
                           key_chunk_size=512, causal_block_size=None, ring_size=1, ring_order=None,
                           grad_dtype=None, workspace=None, out=None, prof_events=None):
    """Gradients (dq, dk, dv) of ringattention given the upstream ``do``.

    Recomputes attention from q, k and the saved ``lse``.  ``grad_dtype``
    defaults to the input dtype (bf16 gradients may be requested as fp32).
    ``out``: optional preallocated (dq, dk, dv); ``prof_events`` as in
    ringattention.
    """
    B, S, H, D = q.shape
    p = _params(S, query_chunk_size, key_chunk_size, causal_block_size, ring_size, ring_order, prof_events)
    gd = q.dtype if grad_dtype is None else grad_dtype
    if out is not None:
        dq, dk, dv = out
    else:
        dq = torch.empty(q.shape, dtype=gd, device=q.device)
        dk = torch.empty(q.shape, dtype=gd, device=q.device)
        dv = torch.empty(q.shape, dtype=gd, device=q.device)
    need = workspace_size(1, q, p, attention_bias is not None, segment_ids is not None)
    if workspace is None or workspace.numel() < need:
        workspace = _workspace(need, q.device)
    ts = [_tensor(x) for x in (q, k, v, o, do, lse)]
    tb, tseg = _tensor(attention_bias), _tensor(segment_ids)
    tdq, tdk, tdv = _tensor(dq), _tensor(dk), _tensor(dv)
    code = load().ra_backward(*[ctypes.byref(x) for x in ts], _ref(tb), _ref(tseg), ctypes.byref(p),
                              ctypes.byref(tdq), ctypes.byref(tdk), ctypes.byref(tdv),
                              None if workspace is None else workspace.data_ptr(), need, _stream())
    check(code, "ra_backward")
    return dq, dk, dv


def ring_step(q_blk, k_blk, v_blk, q_off, k_off, o_acc, m, l, bias_blk=None, seg_q=None, seg_k=None,
              causal_block_size=None):
    """One ring step, updating the running (o_acc, m, l) in place (see ra_step).

    bf16 blocks run on the tensor cores (the forward kernel in ring-step
    mode); fp32 blocks on CUDA cores.  Positions are global: the query block
    starts at token ``q_off``, the visiting key/value block at ``k_off``."""
    p = _params(max(1, q_blk.shape[1]), None, None, causal_block_size, 1, None)
    tq, tk, tv = _tensor(q_blk), _tensor(k_blk), _tensor(v_blk)
    ta, tm, tl = _tensor(o_acc), _tensor(m), _tensor(l)
    tb, tsq, tsk = _tensor(bias_blk), _tensor(seg_q), _tensor(seg_k)
    code = load().ra_step(ctypes.byref(tq), ctypes.byref(tk), ctypes.byref(tv), int(q_off), int(k_off), _ref(tb),
                          _ref(tsq), _ref(tsk), ctypes.byref(p), ctypes.byref(ta), ctypes.byref(tm),
                          ctypes.byref(tl), _stream())
    check(code, "ra_step")


def init_state(B, S, H, D, device):
    """Fresh running state for ring_step: (o_acc = 0, m = -inf, l = 0)."""
    acc = torch.zeros((B, S, H, D), dtype=torch.float32, device=device)
    m = torch.full((B, H, S), float("-inf"), dtype=torch.float32, device=device)
    l = torch.zeros((B, H, S), dtype=torch.float32, device=device)
    return acc, m, l


def finalize(o_acc, m, l, out_dtype=torch.bfloat16, out=None, lse=None):
    """(o_acc, m, l) -> (o, lse).  ``out`` / ``lse``: optional preallocated
    outputs (any strides the C ABI accepts, e.g. views into larger tensors)."""
    B, S, H, D = o_acc.shape
    o = torch.empty((B, S, H, D), dtype=out_dtype, device=o_acc.device) if out is None else out
    if lse is None:
        lse = torch.empty((B, H, S), dtype=torch.float32, device=o_acc.device)
    ta, tm, tl, to, tlse = _tensor(o_acc), _tensor(m), _tensor(l), _tensor(o), _tensor(lse)
    code = load().ra_finalize(ctypes.byref(ta), ctypes.byref(tm), ctypes.byref(tl), ctypes.byref(to),
                              ctypes.byref(tlse), _stream())
    check(code, "ra_finalize")
    return o, lse


def lse_merge(o_a, lse_a, o_b, lse_b, out=None, lse_out=None):
    """Merge two normalised partials over disjoint key sets (out may alias a)."""
    if out is None:
        out = torch.empty_like(o_a)
    if lse_out is None:
        lse_out = torch.empty_like(lse_a)
    ts = [_tensor(x) for x in (o_a, lse_a, o_b, lse_b, out, lse_out)]
    code = load().ra_lse_merge(*[ctypes.byref(x) for x in ts], _stream())
    check(code, "ra_lse_merge")
    return out, lse_out


def blockwise_feedforward(x, w1, w3, w2, chunk_size=4096, out=None, workspace=None):
    """SwiGLU feed-forward y = (silu(x W1^T) * (x W3^T)) W2^T, chunk_size tokens
    at a time (see ra_feedforward).  x: bf16 [T, d_model] (a [..., d_model]
    tensor is flattened); w1, w3: [d_ff, d_model]; w2: [d_model, d_ff]."""
    shape = x.shape
    x2 = x.reshape(-1, shape[-1])
    T, dff = x2.shape[0], w1.shape[0]
    y = torch.empty_like(x2) if out is None else out.reshape(-1, shape[-1])
    lib = load()
    chunk = max(1, min(int(chunk_size), max(T, 1)))
    need = lib.ra_feedforward_workspace_size(chunk, dff)
    if workspace is None or workspace.numel() < need:
        workspace = _workspace(need, x.device)
    ts = [_tensor(t) for t in (x2, w1, w3, w2, y)]
    code = lib.ra_feedforward(*[ctypes.byref(t) for t in ts], chunk, None if workspace is None else workspace.data_ptr(),
                              need, _stream())
    check(code, "ra_feedforward")
    return y.reshape(shape)


def device_status(stream=None) -> int:
    """Synchronize and return (then clear) the device-side status word."""
    s = _stream() if stream is None else stream
    return load().ra_get_device_status(s)


def selftest_timeout(budget_cycles: int = 2_000_000) -> int:
    """Run the bounded-wait failure path on the device and return the status it
    left (RA_ERR_DEVICE_TIMEOUT = 9 when the mechanism works)."""
    check(load().ra_selftest_timeout(int(budget_cycles), _stream()), "ra_selftest_timeout")
    return device_status()


def _host_i32(x):
    if x is None:
        return None, None
    a = torch.as_tensor(x).detach().to("cpu", torch.int32).contiguous()
    return a, a.numpy().ctypes.data_as(ctypes.POINTER(ctypes.c_int32))


def _host_f32(x):
    if x is None:
        return None, None
    a = torch.as_tensor(x).detach().to("cpu", torch.float32).contiguous()
    return a, a.numpy().ctypes.data_as(ctypes.POINTER(ctypes.c_float))


def count_visible_pairs(B, S, H, causal_block_size=None, segment_ids=None, attention_bias=None) -> int:
    """Exact visible (query, key) pair count (host computation in the library)."""
    keep_s, ps = _host_i32(segment_ids)
    keep_b, pb = _host_f32(attention_bias)
    n = load().ra_count_visible_pairs(int(B), int(S), int(H), int(causal_block_size or 0), ps, pb)
    if n < 0:
        raise ValueError("invalid arguments for ra_count_visible_pairs")
    return int(n)


def ring_schedule(S, ring_size, q_first, q_last, causal_block_size=None, ring_order=None, segment_ids=None,
                  attention_bias=None, query_chunk_size=None, key_chunk_size=None):
    """KV tile indices visited, in ring order, by query rows [q_first, q_last] (batch row 0)."""
    p = _params(S, query_chunk_size, key_chunk_size, causal_block_size, ring_size, ring_order)
    keep_s, ps = _host_i32(segment_ids)
    keep_b, pb = _host_f32(attention_bias)
    lib = load()
    n = lib.ra_ring_schedule(int(S), ctypes.byref(p), int(q_first), int(q_last), ps, pb, None, 0)
    if n < 0:
        raise ValueError("invalid arguments for ra_ring_schedule")
    out = (ctypes.c_int32 * max(1, n))()
    lib.ra_ring_schedule(int(S), ctypes.byref(p), int(q_first), int(q_last), ps, pb, out, n)
    return list(out[:n])


class RingAttentionFunction(torch.autograd.Function):
    """autograd wrapper: forward = ra_forward, backward = ra_backward."""

    @staticmethod
    def forward(ctx, q, k, v, attention_bias, segment_ids, kwargs):
        o, lse = ringattention(q, k, v, attention_bias, segment_ids, **kwargs)
        ctx.save_for_backward(q, k, v, o, lse, attention_bias, segment_ids)
        ctx.kwargs = kwargs
        return o

    @staticmethod
    def backward(ctx, do):
        q, k, v, o, lse, bias, seg = ctx.saved_tensors
        dq, dk, dv = ringattention_backward(q, k, v, o, lse, do.contiguous(), bias, seg, **ctx.kwargs)
        return dq, dk, dv, None, None, None


@contextlib.contextmanager
def visible_count_probe(fwd_row_counts=None, bwd_col_counts=None):
    """Inside the block, calls run the debug build of the library, whose
    tensor-core kernels record how many pairs their own skipping and masking
    let into the softmax: per query row in ``fwd_row_counts`` (int32
    [B, H, S], overwritten by each forward) and per key in ``bwd_col_counts``
    (int32 [B, H, S], added to by each backward: zero it first).  For the
    mask bit-exactness tests only."""
    for t in (fwd_row_counts, bwd_col_counts):
        if t is not None and (t.dtype != torch.int32 or not t.is_cuda or not t.is_contiguous()):
            raise ValueError("count buffers must be contiguous int32 CUDA tensors")
    dbg = _lib.load_count()
    check(dbg.ra_debug_set_counts(None if fwd_row_counts is None else fwd_row_counts.data_ptr(),
                                  None if bwd_col_counts is None else bwd_col_counts.data_ptr()),
          "ra_debug_set_counts")
    prev = _lib.swap(dbg)
    try:
        yield
    finally:
        _lib.swap(prev)
        dbg.ra_debug_set_counts(None, None)


class HostStep:
    """One training step (forward + backward) whose inputs and outputs live in
    host memory, through ``ra_train_step_host``: the heads are processed in
    groups, and each group's host->device copy, kernels and device->host copy
    run on three streams so the copies overlap the kernels.

    The object owns the device staging buffers, the workspace and two copy
    streams, sized once for [B, S, H, D] tensors of ``dtype``; call it once
    per step with pinned host tensors.  The kernels run on the caller's
    current stream, which is made to wait for the last copy back."""

    def __init__(self, B, S, H, D, dtype=torch.bfloat16, heads_per_group=None, device=None, has_bias=False,
                 has_segments=False, query_chunk_size=512, key_chunk_size=512, causal_block_size=None,
                 ring_size=1, ring_order=None):
        device = torch.device("cuda") if device is None else torch.device(device)
        if heads_per_group is None:                  # about eight groups: one copy in, one out exposed per step
            heads_per_group = max(1, H // 8)
            while H % heads_per_group:
                heads_per_group -= 1
        self.shape, self.dtype, self.hpg = (B, S, H, D), dtype, int(heads_per_group)
        self.params = _params(S, query_chunk_size, key_chunk_size, causal_block_size, ring_size, ring_order)
        mk = lambda: torch.empty((B, S, H, D), dtype=dtype, device=device)
        self.dev = {n: mk() for n in ("q", "k", "v", "do", "o", "dq", "dk", "dv")}
        self.dev["lse"] = torch.empty((B, H, S), dtype=torch.float32, device=device)
        probe = torch.empty((B, S, self.hpg, D), dtype=dtype, device="meta")
        n = load().ra_workspace_size(1, ctypes.byref(_tensor_meta(probe)), ctypes.byref(self.params),
                                     int(has_bias), int(has_segments))
        self.workspace = _workspace(n, device)
        self.h2d = torch.cuda.Stream(device)
        self.d2h = torch.cuda.Stream(device)

    def __call__(self, q, k, v, do, o, lse, dq, dk, dv, attention_bias=None, segment_ids=None):
        """q, k, v, do: host [B,S,H,D]; o, dq, dk, dv: host outputs like q; lse: host fp32 [B,H,S].
        attention_bias / segment_ids: device tensors or None."""
        for x in (q, k, v, do, o, lse, dq, dk, dv):
            if x.is_cuda:
                raise ValueError("HostStep takes host tensors (pinned for overlap)")
        t = RaHostStep()
        for name, x in (("q", q), ("k", k), ("v", v), ("d_o", do), ("o", o), ("lse", lse), ("dq", dq), ("dk", dk),
                        ("dv", dv)):
            setattr(t, name, _tensor(x))
        for name, key in (("dev_q", "q"), ("dev_k", "k"), ("dev_v", "v"), ("dev_do", "do"), ("dev_o", "o"),
                          ("dev_lse", "lse"), ("dev_dq", "dq"), ("dev_dk", "dk"), ("dev_dv", "dv")):
            setattr(t, name, _tensor(self.dev[key]))
        ws = self.workspace
        code = load().ra_train_step_host(ctypes.byref(t), _ref(_tensor(attention_bias)), _ref(_tensor(segment_ids)),
                                         ctypes.byref(self.params), self.hpg, 0 if ws is None else ws.data_ptr(),
                                         0 if ws is None else ws.numel(), _stream(), self.h2d.cuda_stream,
                                         self.d2h.cuda_stream)
        check(code, "ra_train_step_host")


def _tensor_meta(t: torch.Tensor) -> RaTensor:
    """Shape-only descriptor (no data) for size queries."""
    r = RaTensor()
    r.data = 0
    r.dtype = _DT[t.dtype]
    r.ndim = t.dim()
    for i in range(t.dim()):
        r.shape[i] = t.shape[i]
        r.stride[i] = t.stride(i)
    return r
