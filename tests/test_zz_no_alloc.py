"""ra_forward_static: the forward entry point that allocates nothing.

Some callers cannot allocate device memory (a host program that links only
this library and has no device allocator of its own, or code running under a
fixed memory budget where an allocation could fail or synchronize the
device).  For them the library keeps its forward scratch in one static device
array.  This test calls that entry point through the C ABI, twice in a row
(the array keeps the previous call's contents), and checks its outputs
against ra_forward with a caller-allocated workspace, within the bf16
tolerance the other parity tests use.  It lives in its own file, collected
last, and passes alone in a fresh process as well as after the other tests.
"""

from __future__ import annotations

import ctypes

import pytest
import torch

import workloads as W
from checker import compare
from gpu_util import to64

pytestmark = pytest.mark.gpu

ra = pytest.importorskip("long_context_exact_ordered_b200")
from long_context_exact_ordered_b200 import _lib, api  # noqa: E402


def _call_static(inp, w, o, lse):
    p = api._params(w.S, w.chunk, w.chunk, w.causal_block_size, w.P, None)
    ts = [api._tensor(x) for x in (inp["q"], inp["k"], inp["v"])]
    tb, tsg = api._tensor(inp["bias"]), api._tensor(inp["seg"])
    to, tl = api._tensor(o), api._tensor(lse)
    return _lib.load().ra_forward_static(*[ctypes.byref(x) for x in ts], api._ref(tb), api._ref(tsg),
                                         ctypes.byref(p), ctypes.byref(to), ctypes.byref(tl),
                                         torch.cuda.current_stream().cuda_stream)


CASES = [
    # (workload, random bias with -inf keys)
    (dict(B=2, H=2, D=128, S=1024, P=4, chunk=256, causal_block_size=1, segments="packed", doc_lo=40, doc_hi=300,
          seed=31), True),
    (dict(B=1, H=3, D=64, S=640, P=5, chunk=128, causal_block_size=None, segments="packed", doc_lo=50, doc_hi=200,
          seed=32), True),
    # neither bias nor segments: no scratch is needed and none is looked up
    (dict(B=1, H=2, D=128, S=768, P=3, chunk=256, causal_block_size=1, seed=33), False),
    # fp32 inputs (CUDA-core path) with segment metadata in the static array
    (dict(B=1, H=2, D=64, S=512, P=2, chunk=256, causal_block_size=1, dtype="f32", segments="packed", doc_lo=40,
          doc_hi=200, seed=34), False),
]


@pytest.mark.parametrize("case", CASES, ids=["bf16-D128-seg-bias", "bf16-D64-seg-bias", "bf16-plain", "f32-seg"])
def test_static_scratch_forward_matches_workspace_forward_twice(case):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda:0")
    spec, with_bias = case
    w = W.small_workload(**spec)
    inp = W.make_inputs(w, dev)
    if with_bias:
        g = torch.Generator(device="cpu").manual_seed(w.seed)
        bias = torch.randn((w.B, w.S), generator=g)
        bias[:, torch.randint(0, w.S, (w.S // 7,), generator=g)] = float("-inf")
        inp["bias"] = bias.to(dev)
    ref_o, ref_lse = ra.ringattention(inp["q"], inp["k"], inp["v"], inp["bias"], inp["seg"],
                                      query_chunk_size=w.chunk, key_chunk_size=w.chunk,
                                      causal_block_size=w.causal_block_size, ring_size=w.P)
    kind = "f32" if w.dtype == "f32" else "bf16"
    for _ in range(2):                                   # two calls in a row share the static array
        o = torch.full_like(inp["q"], float("nan"))
        lse = torch.full((w.B, w.H, w.S), float("nan"), dtype=torch.float32, device=dev)
        assert _call_static(inp, w, o, lse) == 0
        torch.cuda.synchronize()
        assert ra.device_status() == 0
        res = compare(to64(o), to64(ref_o), kind)
        assert res.ok, str(res)
        assert torch.equal(o, ref_o) and torch.equal(lse, ref_lse)


def test_static_scratch_rejects_oversized_problems():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    t = _lib.RaTensor()
    t.data = 0x10000
    t.dtype = _lib.RA_BF16
    t.ndim = 4
    shape = [65, 131072, 1, 128]                              # 65 * 1024 tiles > 65536
    for i, s in enumerate(shape):
        t.shape[i] = s
    seg = _lib.RaTensor()
    seg.data = 0x10000
    seg.dtype = _lib.RA_I32
    seg.ndim = 2
    seg.shape[0], seg.shape[1] = 65, 131072
    p = api._params(131072, 512, 512, 1, 8, None)
    code = _lib.load().ra_forward_static(ctypes.byref(t), ctypes.byref(t), ctypes.byref(t), None, ctypes.byref(seg),
                                         ctypes.byref(p), ctypes.byref(t), ctypes.byref(t), None)
    assert code == 11        # RA_ERR_STATIC_LIMIT, before any device work
