"""Forward parity of the CUDA path against the float64 oracle (needs a B200).

Tolerances (checker.py): bf16 outputs max-abs excess over half a bf16 ulp
<= 1e-2 and mean-abs <= 1e-3; fp32 outputs max-abs <= 1e-5; LSE (fp32) max-abs
<= 1e-3 on the bf16 path and <= 1e-5 on the fp32 path; integer counts exact.
"""

from __future__ import annotations

import itertools

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from checker import compare
from gpu_util import gather_rows, oracle_full, oracle_rows, to64, to_np

pytestmark = pytest.mark.gpu

ra = pytest.importorskip("long_context_exact_ordered_b200")

LSE_BF16 = 1e-3
LSE_F32 = 1e-5


def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def run(inp, w, **kw):
    args = dict(query_chunk_size=w.chunk, key_chunk_size=w.chunk, causal_block_size=w.causal_block_size,
                ring_size=w.P)
    args.update(kw)
    return ra.ringattention(inp["q"], inp["k"], inp["v"], inp.get("bias"), inp.get("seg"), **args)


def assert_lse(got, want, tol):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    both = np.isneginf(got) & np.isneginf(want)
    with np.errstate(invalid="ignore"):          # -inf - -inf where both rows are empty
        err = np.where(both, 0.0, np.abs(got - want))
    assert np.all(np.isfinite(err)), "lse -inf pattern differs"
    assert err.max() <= tol, f"lse max abs err {err.max():.3e} > {tol}"


def test_tiny_fp32_config_full():
    w = W.WORKLOADS["tiny"]
    inp = W.make_inputs(w, dev())
    o, lse = run(inp, w)
    ro, rl = oracle_full(inp, w.causal_block_size)
    res = compare(to64(o), ro, "f32")
    assert res.ok, str(res)
    assert_lse(to64(lse), rl, LSE_F32)
    assert ra.device_status() == 0


SMALL = [
    # D,   S,    P, c,    segments, bias,   B, H
    (64, 512, 2, 1, None, None, 1, 2),
    (128, 512, 2, 1, None, None, 1, 2),
    (128, 384, 3, None, None, None, 1, 2),      # odd number of query tiles
    (128, 1000, 2, 1, None, None, 1, 1),        # ragged last tile
    (64, 1024, 4, 3, None, None, 2, 1),         # block-causal
    (128, 1024, 4, 1, "packed", None, 1, 2),    # packed documents
    (64, 768, 2, None, None, "neginf", 1, 3),   # additive bias with masked keys
    (128, 640, 5, 1, "packed", "neginf", 2, 2),
    (64, 2048, 8, 1, None, "zeros", 1, 2),
    (128, 130, 1, 1, None, None, 1, 1),         # one full tile plus 2 tokens
]


def make_small(D, S, P, c, segments, bias, B, H, dtype="bf16", seed=11):
    w = W.small_workload(B=B, H=H, D=D, S=S, P=P, chunk=S // P, causal_block_size=c, dtype=dtype,
                         segments=segments, bias="zeros" if bias == "zeros" else None, seed=seed,
                         doc_lo=40, doc_hi=300)
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


@pytest.mark.parametrize("case", SMALL, ids=lambda c: "D{}-S{}-P{}-c{}-{}-{}-B{}H{}".format(*c))
def test_bf16_small_full_parity(case):
    w, inp = make_small(*case)
    o, lse = run(inp, w)
    ro, rl = oracle_full(inp, w.causal_block_size)
    res = compare(to64(o), ro, "bf16")
    assert res.ok, str(res)
    assert_lse(to64(lse), rl, LSE_BF16)
    assert ra.device_status() == 0


RAMP = [
    # D,   S,    P, c,    segments, bias,   B, H
    (64, 1024, 2, 1, None, "ramp", 1, 2),
    (64, 1024, 2, None, None, "ramp", 1, 2),
    (128, 1024, 2, 1, None, "ramp", 1, 2),
    (64, 1024, 4, 1, "packed", "ramp", 1, 2),
]


@pytest.mark.parametrize("case", RAMP, ids=lambda c: "D{}-S{}-P{}-c{}-{}-{}-B{}H{}".format(*c))
def test_reference_moves_inside_tiles(case):
    """Scores that keep growing along the keys (a bias ramp of ~9 log2 units
    per half tile) move the softmax's running reference at every key tile,
    so every tile takes the rescale of O and of the running sum."""
    w, inp = make_small(*case)
    o, lse = run(inp, w)
    ro, rl = oracle_full(inp, w.causal_block_size)
    res = compare(to64(o), ro, "bf16")
    assert res.ok, str(res)
    assert_lse(to64(lse), rl, LSE_BF16)
    assert ra.device_status() == 0


@pytest.mark.parametrize("case", [SMALL[1], SMALL[5]], ids=["causal", "packed"])
def test_fp32_small_full_parity(case):
    w, inp = make_small(*case, dtype="f32")
    o, lse = run(inp, w)
    ro, rl = oracle_full(inp, w.causal_block_size)
    res = compare(to64(o), ro, "f32")
    assert res.ok, str(res)
    assert_lse(to64(lse), rl, LSE_F32)


def test_ring_order_invariance_all_permutations():
    w, inp = make_small(128, 1024, 4, 1, "packed", None, 1, 2)
    base, bl = run(inp, w)
    ro, rl = oracle_full(inp, 1)
    for perm in itertools.permutations(range(4)):
        o, lse = run(inp, w, ring_order=list(perm))
        assert compare(to64(o), ro, "bf16").ok
        assert float((o.float() - base.float()).abs().max()) <= 1e-3 + 2 ** -8 * float(base.float().abs().max())
        assert_lse(to64(lse), rl, LSE_BF16)


def test_chunk_size_does_not_change_result():
    w, inp = make_small(128, 2048, 2, 1, None, None, 1, 2)
    base, bl = run(inp, w)
    for qc, kc in [(128, 128), (256, 512), (1024, 1024), (512, 128)]:
        o, lse = run(inp, w, query_chunk_size=qc, key_chunk_size=kc)
        assert torch.equal(o, base) and torch.equal(lse, bl)


def test_forward_is_deterministic():
    w, inp = make_small(128, 1024, 4, 1, "packed", "neginf", 2, 2)
    a, la = run(inp, w)
    b, lb = run(inp, w)
    assert torch.equal(a, b) and torch.equal(la, lb)


@pytest.mark.parametrize("segments", [None, "packed"])
def test_zero_queries_give_visible_means_and_exact_counts(segments):
    """q = 0, bias = 0: o_i = mean of visible v_j and exp(lse_i) = number of visible keys."""
    w, inp = make_small(128, 1536, 4, 1, segments, None, 1, 2)
    inp["q"] = torch.zeros_like(inp["q"])
    o, lse = run(inp, w)
    ro, rl = oracle_full(inp, 1)
    assert compare(to64(o), ro, "bf16").ok
    seg = None if inp["seg"] is None else to_np(inp["seg"])[0]
    n_vis = oracle.visible_count_rows(np.arange(w.S), w.S, 1, seg)
    got = np.rint(np.exp(to64(lse)[0]))
    for h in range(w.H):
        np.testing.assert_array_equal(got[h], n_vis)


def test_single_visible_key_rows_are_exact():
    w, inp = make_small(64, 512, 2, 1, "packed", None, 1, 2)
    o, lse = run(inp, w)
    seg = to_np(inp["seg"])[0]
    starts = np.nonzero(np.r_[True, seg[1:] != seg[:-1]])[0]
    for i in starts:   # causal row i = first of its segment sees only key i
        assert torch.equal(o[0, i], inp["v"][0, i])


def test_fully_masked_rows_give_zero_and_neg_inf():
    w, inp = make_small(128, 256, 1, 1, None, None, 1, 2)
    bias = torch.zeros((1, 256), device=dev())
    bias[0, :3] = float("-inf")         # rows 0..2 see no key under causal masking
    inp["bias"] = bias
    o, lse = run(inp, w)
    assert torch.all(o[0, :3] == 0)
    assert torch.all(torch.isneginf(lse[0, :, :3]))
    ro, rl = oracle_full(inp, 1)
    assert compare(to64(o), ro, "bf16").ok


def test_step_finalize_merge_follow_the_ring():
    """Drive the fp32 ra_step over the ring by hand, then finalize / merge partials,
    held to the fp32 bound 1e-5 (the bf16 tensor-core step is tested in
    test_gpu_step.py under the bf16 rule)."""
    for dtype in ("f32",):
        w, inp = make_small(64, 1024, 4, 1, "packed", "neginf", 1, 2, dtype=dtype)
        q, k, v, bias, seg = inp["q"], inp["k"], inp["v"], inp["bias"], inp["seg"]
        blk = w.S // w.P
        ro, rl = oracle_full(inp, 1)
        outs, lses = [], []
        for r in range(w.P):                      # virtual rank r
            qs = slice(r * blk, (r + 1) * blk)
            acc, m, l = ra.init_state(1, blk, w.H, w.D, q.device)
            for t in range(w.P):                  # step t: KV block (r - t) mod P
                src = (r - t) % w.P
                ks = slice(src * blk, (src + 1) * blk)
                ra.ring_step(q[:, qs], k[:, ks], v[:, ks], r * blk, src * blk, acc, m, l,
                             bias_blk=bias[:, ks].contiguous(), seg_q=seg[:, qs].contiguous(),
                             seg_k=seg[:, ks].contiguous(), causal_block_size=1)
            o, lse = ra.finalize(acc, m, l, torch.float32)
            outs.append(o)
            lses.append(lse)
        o = torch.cat(outs, 1)
        lse = torch.cat(lses, 2)
        assert compare(to64(o), ro, "f32").ok
        assert_lse(to64(lse), rl, LSE_F32)
        # merge: partial over keys of the first half + partial over the second half
        half = w.S // 2
        parts = []
        for lo, hi in ((0, half), (half, w.S)):
            acc, m, l = ra.init_state(1, w.S, w.H, w.D, q.device)
            ra.ring_step(q, k[:, lo:hi], v[:, lo:hi], 0, lo, acc, m, l, bias_blk=bias[:, lo:hi].contiguous(),
                         seg_q=seg, seg_k=seg[:, lo:hi].contiguous(), causal_block_size=1)
            parts.append(ra.finalize(acc, m, l, torch.float32))
        mo, ml = ra.lse_merge(parts[0][0], parts[0][1], parts[1][0], parts[1][1])
        assert compare(to64(mo), ro, "f32").ok
        assert_lse(to64(ml), rl, LSE_F32)


# ---------------------------------------------------------------- full-size configs

def _full_config(name, n_rows=4096):
    w = W.WORKLOADS[name]
    inp = W.make_inputs(w, dev(), with_grad_output=False)
    o, lse = run(inp, w)
    torch.cuda.synchronize()
    assert ra.device_status() == 0
    samples = W.sample_rows(w, None if inp["seg"] is None else to_np(inp["seg"]), n=n_rows)
    go, gl = gather_rows(o, lse, samples)
    ro, rl = oracle_rows(inp, samples, w.causal_block_size)
    res = compare(go, ro, "bf16")
    assert res.ok, f"{name}: {res}"
    assert_lse(gl, rl, LSE_BF16)
    return o, lse


@pytest.mark.slow
def test_config_noncausal32k():
    _full_config("noncausal32k")


@pytest.mark.slow
def test_config_packed128k():
    _full_config("packed128k")


@pytest.mark.slow
def test_config_causal1m():
    o, lse = _full_config("causal1m")
    del o, lse
    torch.cuda.empty_cache()
