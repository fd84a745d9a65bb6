"""The per-step entry (ra_step) on the tensor cores, driven round the ring by hand.

For bf16 inputs ra_step runs the forward kernel in ring-step mode: the query
block of virtual rank r meets one visiting key/value block per call and the
block's partial is merged into the caller's fp32 running state (m, l,
o_acc).  Driving it over every step of the ring ("Ring Attention技术解析"
§2.2: at step t rank r holds the block that started t ranks behind it) and
finalizing must give exact attention: the oracle's float64 result within the
bf16 rule of checker.py (O rounded to bf16 at the end), LSE within 1e-3.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import workloads as W
from checker import compare
from gpu_util import oracle_full, to64

pytestmark = pytest.mark.gpu
ra = pytest.importorskip("long_context_exact_ordered_b200")

LSE_BF16 = 1e-3


def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def make(D, S, P, c, segments, bias, B, H, seed=51):
    w = W.small_workload(B=B, H=H, D=D, S=S, P=P, chunk=S // P, causal_block_size=c, segments=segments,
                         seed=seed, doc_lo=40, doc_hi=300)
    inp = W.make_inputs(w, dev())
    if bias == "neginf":
        g = torch.Generator(device="cpu").manual_seed(seed + 1)
        b = torch.randn((B, S), generator=g)
        b[:, torch.randint(0, S, (S // 5,), generator=g)] = float("-inf")
        inp["bias"] = b.to(dev())
    elif bias == "ramp":
        # scores grow along the keys by ~9 (log2 units) per half tile: the
        # softmax reference must move inside every key tile
        inp["bias"] = (0.1 * torch.arange(S, dtype=torch.float32)).expand(B, S).contiguous().to(dev())
    return w, inp


def ring_by_steps(w, inp, order=None, out_dtype=torch.bfloat16):
    """Every virtual rank r runs ra_step for t = 0..P-1 against block (r - order[t]) mod P."""
    q, k, v, bias, seg = inp["q"], inp["k"], inp["v"], inp["bias"], inp["seg"]
    P, blk = w.P, w.S // w.P
    order = list(range(P)) if order is None else order
    outs, lses = [], []
    for r in range(P):
        qs = slice(r * blk, (r + 1) * blk)
        acc, m, l = ra.init_state(w.B, blk, w.H, w.D, q.device)
        for t in range(P):
            src = (r - order[t]) % P
            ks = slice(src * blk, (src + 1) * blk)
            ra.ring_step(q[:, qs], k[:, ks], v[:, ks], r * blk, src * blk, acc, m, l,
                         bias_blk=None if bias is None else bias[:, ks].contiguous(),
                         seg_q=None if seg is None else seg[:, qs].contiguous(),
                         seg_k=None if seg is None else seg[:, ks].contiguous(),
                         causal_block_size=w.causal_block_size)
        o, lse = ra.finalize(acc, m, l, out_dtype)
        outs.append(o)
        lses.append(lse)
    torch.cuda.synchronize()
    assert ra.device_status() == 0
    return torch.cat(outs, 1), torch.cat(lses, 2)


def assert_lse(got, want, tol):
    both = np.isneginf(got) & np.isneginf(want)
    with np.errstate(invalid="ignore"):
        err = np.where(both, 0.0, np.abs(got - want))
    assert np.all(np.isfinite(err)), "lse -inf pattern differs"
    assert err.max() <= tol, f"lse max abs err {err.max():.3e}"


CASES = [
    # D,  S,    P, c,    segments, bias,    B, H
    (128, 1024, 4, 1, None, None, 1, 2),
    (64, 1024, 4, 1, None, None, 1, 2),
    (128, 1000, 4, 1, None, None, 1, 2),          # blocks of 250 tokens: ragged query and key tiles
    (128, 1536, 3, None, None, None, 2, 1),       # non-causal: every step sees its whole block
    (128, 1536, 3, 3, "packed", None, 1, 2),      # block-causal, packed documents
    (128, 640, 5, 1, "packed", "neginf", 2, 2),   # segments and a bias with masked keys
    (64, 768, 2, None, None, "neginf", 1, 3),
    (128, 8192, 2, 1, "packed", None, 1, 2),      # 4096-token blocks: many tiles per step
    (64, 1024, 4, 1, None, "ramp", 1, 2),         # the softmax reference moves at every key tile
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "D{}-S{}-P{}-c{}-{}-{}-B{}H{}".format(*c))
def test_bf16_step_follows_the_ring(case):
    w, inp = make(*case)
    o, lse = ring_by_steps(w, inp)
    ro, rl = oracle_full(inp, w.causal_block_size)
    res = compare(to64(o), ro, "bf16")
    assert res.ok, str(res)
    assert_lse(to64(lse), rl, LSE_BF16)


def test_bf16_step_order_does_not_matter():
    w, inp = make(128, 1024, 4, 1, "packed", "neginf", 1, 2)
    ro, rl = oracle_full(inp, 1)
    for order in ([3, 1, 0, 2], [2, 3, 1, 0]):
        o, lse = ring_by_steps(w, inp, order)
        assert compare(to64(o), ro, "bf16").ok
        assert_lse(to64(lse), rl, LSE_BF16)


def test_bf16_step_hidden_block_leaves_state_unchanged():
    """A causal step whose whole key block lies after the query block changes nothing."""
    w, inp = make(128, 1024, 4, 1, None, None, 1, 2)
    q, k, v = inp["q"], inp["k"], inp["v"]
    acc, m, l = ra.init_state(1, 256, 2, 128, q.device)
    ra.ring_step(q[:, 256:512], k[:, 256:512], v[:, 256:512], 256, 256, acc, m, l, causal_block_size=1)
    before = (acc.clone(), m.clone(), l.clone())
    ra.ring_step(q[:, 256:512], k[:, 768:1024], v[:, 768:1024], 256, 768, acc, m, l, causal_block_size=1)
    torch.cuda.synchronize()
    for a, b in zip(before, (acc, m, l)):
        assert torch.equal(a, b)


def test_bf16_step_agrees_with_fused_forward():
    """The step route and the fused ring kernel compute the same attention."""
    w, inp = make(128, 2048, 4, 1, "packed", None, 1, 4)
    o_s, l_s = ring_by_steps(w, inp, out_dtype=torch.float32)
    o_f, l_f = ra.ringattention(inp["q"], inp["k"], inp["v"], None, inp["seg"], query_chunk_size=512,
                                key_chunk_size=512, causal_block_size=1, ring_size=4)
    # fused O is bf16-rounded; the step route's fp32 O is within half a bf16 ulp + 1e-2 of it
    assert compare(to64(o_s), to64(o_f), "bf16").ok
    assert_lse(to64(l_s), to64(l_f), LSE_BF16)
