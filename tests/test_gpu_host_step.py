"""The host-buffer training step (ra_train_step_host / HostStep) on a B200.

Per group of heads it runs exactly ra_forward then ra_backward, so its
results must equal those calls on the whole device tensors: O, LSE, dK and dV
bit for bit; dQ within rounding (its fp32 partial sums are added in no fixed
order).  It is also held to the float64 oracle like the device API.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from checker import compare, operand_rounding_bound
from gpu_util import to64, to_np

pytestmark = pytest.mark.gpu
ra = pytest.importorskip("long_context_exact_ordered_b200")


def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def pinned_like(t):
    return torch.empty(t.shape, dtype=t.dtype, pin_memory=True)


CASES = [
    # D, S, P, c, segments, bias, B, H, heads_per_group, dtype
    (128, 1024, 4, 1, None, None, 1, 4, 2, "bf16"),
    (128, 640, 5, 1, "packed", "neginf", 2, 4, 1, "bf16"),
    (128, 768, 2, None, None, None, 1, 6, 3, "bf16"),
    (64, 512, 2, 1, "packed", None, 1, 4, 2, "bf16"),
    (128, 512, 2, 1, None, None, 1, 2, 1, "f32"),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "D{}-S{}-P{}-c{}-{}-{}-B{}H{}-g{}-{}".format(*c))
def test_host_step_equals_device_calls(case):
    D, S, P, c, segments, bias, B, H, hpg, dtype = case
    w = W.small_workload(B=B, H=H, D=D, S=S, P=P, chunk=S // P, causal_block_size=c, dtype=dtype, segments=segments,
                         seed=41, doc_lo=40, doc_hi=300, backward=True)
    inp = W.make_inputs(w, dev())
    if bias == "neginf":
        g = torch.Generator(device="cpu").manual_seed(42)
        b = torch.randn((B, S), generator=g)
        b[:, torch.randint(0, S, (S // 5,), generator=g)] = float("-inf")
        inp["bias"] = b.to(dev())
    kw = dict(query_chunk_size=w.chunk, key_chunk_size=w.chunk, causal_block_size=c, ring_size=P)
    # device API
    o_d, lse_d = ra.ringattention(inp["q"], inp["k"], inp["v"], inp["bias"], inp["seg"], **kw)
    dq_d, dk_d, dv_d = ra.ringattention_backward(inp["q"], inp["k"], inp["v"], o_d, lse_d, inp["do"], inp["bias"],
                                                 inp["seg"], **kw)
    # host API
    host = {n: inp[n].cpu().pin_memory() for n in ("q", "k", "v", "do")}
    outs = {n: pinned_like(host["q"]) for n in ("o", "dq", "dk", "dv")}
    lse_h = torch.empty((B, H, S), dtype=torch.float32, pin_memory=True)
    step = ra.HostStep(B, S, H, D, dtype=inp["q"].dtype, heads_per_group=hpg, device=dev(),
                       has_bias=inp["bias"] is not None, has_segments=inp["seg"] is not None, **kw)
    step(host["q"], host["k"], host["v"], host["do"], outs["o"], lse_h, outs["dq"], outs["dk"], outs["dv"],
         attention_bias=inp["bias"], segment_ids=inp["seg"])
    torch.cuda.synchronize()
    assert ra.device_status() == 0
    for name, got, want in (("o", outs["o"], o_d), ("lse", lse_h, lse_d), ("dk", outs["dk"], dk_d),
                            ("dv", outs["dv"], dv_d)):
        assert torch.equal(got, want.cpu()), name
    # dQ: the same values up to the order of the fp32 partial sums (one output ulp)
    a64, b64 = to64(outs["dq"]), to64(dq_d)
    rel = 2.0 ** -7 if dtype == "bf16" else 1e-5
    assert np.all(np.abs(a64 - b64) <= np.abs(b64) * rel + 1e-6), "dq vs device API"
    # and the oracle, through the same rules as the device API's tests: cases with
    # a random bias allow each bf16 gradient element the exact bound of the bf16
    # rounding of the P and dS operands (checker.py)
    args = [to64(inp[n]) for n in ("q", "k", "v", "do")]
    bias64, seg = to64(inp["bias"]), to_np(inp["seg"])
    ro, rl = oracle.attention_forward(*args[:3], bias64, seg, c)
    stored = torch.from_numpy(ro).to(inp["q"].dtype).double().numpy()
    rq, rk, rv = oracle.attention_backward(*args, bias64, seg, c, o=stored, lse=rl)
    bounds = (None, None, None)
    if bias is not None and dtype == "bf16":
        mags = oracle.backward_term_magnitudes(*args, bias64, seg, c, o=stored, lse=rl)
        bounds = tuple(operand_rounding_bound(m, S) for m in mags)
    kind = "bf16" if dtype == "bf16" else "f32"
    tol = {} if dtype == "bf16" else {"max_abs": 1e-4}
    for name, got, want, bnd in (("dq", outs["dq"], rq, bounds[0]), ("dk", outs["dk"], rk, bounds[1]),
                                 ("dv", outs["dv"], rv, bounds[2])):
        extra = dict(tol) if bnd is None else dict(tol, rounding_bound=bnd)
        res = compare(to64(got), want, kind, **extra)
        assert res.ok, f"{name} vs oracle: {res}"


def test_host_step_repeats_and_reuses_buffers():
    """Two back-to-back steps with different inputs on the same HostStep."""
    w = W.small_workload(B=1, H=4, D=128, S=1024, P=4, chunk=256, causal_block_size=1, seed=43, backward=True)
    kw = dict(query_chunk_size=256, key_chunk_size=256, causal_block_size=1, ring_size=4)
    step = ra.HostStep(1, 1024, 4, 128, heads_per_group=1, device=dev(), **kw)
    results = []
    for seed in (43, 44):
        inp = W.make_inputs(W.small_workload(B=1, H=4, D=128, S=1024, P=4, chunk=256, causal_block_size=1, seed=seed,
                                             backward=True), dev())
        host = {n: inp[n].cpu().pin_memory() for n in ("q", "k", "v", "do")}
        outs = {n: pinned_like(host["q"]) for n in ("o", "dq", "dk", "dv")}
        lse_h = torch.empty((1, 4, 1024), dtype=torch.float32, pin_memory=True)
        step(host["q"], host["k"], host["v"], host["do"], outs["o"], lse_h, outs["dq"], outs["dk"], outs["dv"])
        results.append((inp, outs, lse_h))
    torch.cuda.synchronize()
    for inp, outs, lse_h in results:
        o_d, lse_d = ra.ringattention(inp["q"], inp["k"], inp["v"], None, None, **kw)
        assert torch.equal(outs["o"], o_d.cpu()) and torch.equal(lse_h, lse_d.cpu())
    assert not torch.equal(results[0][1]["o"], results[1][1]["o"])
