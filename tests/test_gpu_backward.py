"""Backward parity of the CUDA path against the float64 oracle (needs a B200).

The backward receives the forward output as stored (bf16 for bf16 inputs)
and forms Delta_i = <dO_i, o_i> from it, so the oracle's reference gradient
takes Delta from its own float64 output rounded (nearest even) to the input
dtype.

dQ, dK, dV: bf16 outputs use the bf16 rule of checker.py (max-abs excess over
half a bf16 ulp <= 1e-2, mean-abs <= 1e-3).  Cases with a random additive
bias draw it from N(0, 1) with a fifth of the keys masked (-inf): a few keys
then carry most of the attention of many rows, and the bf16 rounding of the
P and dS operands can move a gradient element by more than 1e-2; those cases
allow each element the exact bound of that rounding,
max(1e-2, operand_rounding_bound(backward_term_magnitudes)) (checker.py).
fp32 gradient outputs of bf16 inputs use the raw max-abs 1e-2 / mean-abs
1e-3; fp32 inputs (CUDA-core path) use max-abs 1e-4 (gradients sum many more
terms than the forward).
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from checker import compare, operand_rounding_bound
from gpu_util import gather_rows, oracle_rows, to64, to_np

pytestmark = pytest.mark.gpu
ra = pytest.importorskip("long_context_exact_ordered_b200")


def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def kw(w, **extra):
    d = dict(query_chunk_size=w.chunk, key_chunk_size=w.chunk, causal_block_size=w.causal_block_size,
             ring_size=w.P)
    d.update(extra)
    return d


def make(D, S, P, c, segments, bias, B, H, dtype="bf16", seed=21):
    w = W.small_workload(B=B, H=H, D=D, S=S, P=P, chunk=S // P, causal_block_size=c, dtype=dtype,
                         segments=segments, seed=seed, doc_lo=40, doc_hi=300, backward=True)
    inp = W.make_inputs(w, dev())
    if bias == "neginf":
        g = torch.Generator(device="cpu").manual_seed(seed + 1)
        b = torch.randn((B, S), generator=g)
        b[:, torch.randint(0, S, (S // 5,), generator=g)] = float("-inf")
        inp["bias"] = b.to(dev())
    return w, inp


def run_both(w, inp, grad_dtype=None, **extra):
    o, lse = ra.ringattention(inp["q"], inp["k"], inp["v"], inp["bias"], inp["seg"], **kw(w, **extra))
    g = ra.ringattention_backward(inp["q"], inp["k"], inp["v"], o, lse, inp["do"], inp["bias"], inp["seg"],
                                  grad_dtype=grad_dtype, **kw(w, **extra))
    torch.cuda.synchronize()
    assert ra.device_status() == 0
    return o, lse, g


def stored(o64, dtype):
    """The forward output as the library stores it: rounded to nearest even in `dtype`."""
    return torch.from_numpy(o64).to(dtype).double().numpy()


def oracle_grads(inp, c, bounds=False):
    """Oracle gradients (dq, dk, dv); with ``bounds``, also the per-element
    operand rounding bounds of the three gradients (checker.py)."""
    args = [to64(inp[n]) for n in ("q", "k", "v", "do")]
    bias, seg = to64(inp["bias"]), to_np(inp["seg"])
    o, lse = oracle.attention_forward(*args[:3], bias, seg, c)
    o_st = stored(o, inp["q"].dtype)
    grads = oracle.attention_backward(*args, bias, seg, c, o=o_st, lse=lse)
    if not bounds:
        return grads
    S = args[0].shape[1]
    mags = oracle.backward_term_magnitudes(*args, bias, seg, c, o=o_st, lse=lse)
    return grads, tuple(operand_rounding_bound(m, S) for m in mags)


CASES = [
    # D,  S,    P, c,    segments, bias,   B, H
    (128, 512, 2, 1, None, None, 1, 2),
    (128, 384, 3, None, None, None, 1, 2),       # odd tiles, non-causal
    (128, 1000, 2, 1, None, None, 1, 1),         # ragged
    (128, 1024, 4, 3, None, None, 2, 1),         # block-causal
    (128, 1024, 4, 1, "packed", None, 1, 2),
    (128, 640, 5, 1, "packed", "neginf", 2, 2),
    (128, 768, 2, None, None, "neginf", 1, 2),
    (64, 512, 2, 1, "packed", None, 1, 2),       # head_dim 64 (tensor cores, zero-padded dQ^T)
    (64, 1000, 4, None, None, "neginf", 2, 2),   # head_dim 64, ragged, non-causal, masked keys
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "D{}-S{}-P{}-c{}-{}-{}-B{}H{}".format(*c))
def test_bf16_backward_full_parity(case):
    w, inp = make(*case)
    o, lse, (dq, dk, dv) = run_both(w, inp)
    if inp["bias"] is None:
        rq, rk, rv = oracle_grads(inp, w.causal_block_size)
        bq = bk = bv = None
    else:
        (rq, rk, rv), (bq, bk, bv) = oracle_grads(inp, w.causal_block_size, bounds=True)
    for name, g, r, bnd in (("dq", dq, rq, bq), ("dk", dk, rk, bk), ("dv", dv, rv, bv)):
        res = compare(to64(g), r, "bf16", rounding_bound=bnd)
        assert res.ok, f"{name}: {res}"


@pytest.mark.parametrize("D", [128, 64])
def test_fp32_gradients_of_bf16_inputs_raw_tolerance(D):
    w, inp = make(D, 1024, 4, 1, "packed", None, 1, 2)
    o, lse, (dq, dk, dv) = run_both(w, inp, grad_dtype=torch.float32)
    assert dq.dtype == torch.float32
    rq, rk, rv = oracle_grads(inp, 1)
    for name, g, r in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        res = compare(to64(g), r, "f32", max_abs=1e-2, mean_abs=1e-3)
        assert res.ok, f"{name}: {res}"


@pytest.mark.parametrize("case", [CASES[0], CASES[4]], ids=["causal", "packed"])
def test_fp32_inputs_backward(case):
    w, inp = make(*case, dtype="f32")
    o, lse, (dq, dk, dv) = run_both(w, inp)
    rq, rk, rv = oracle_grads(inp, w.causal_block_size)
    for name, g, r in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        res = compare(to64(g), r, "f32", max_abs=1e-4)
        assert res.ok, f"{name}: {res}"


def test_backward_ring_order_and_determinism():
    w, inp = make(128, 1024, 4, 1, "packed", None, 1, 2)
    _, _, (dq0, dk0, dv0) = run_both(w, inp)
    _, _, (dq1, dk1, dv1) = run_both(w, inp)
    assert torch.equal(dk0, dk1) and torch.equal(dv0, dv1)        # no atomics on dK / dV
    assert float((dq0.float() - dq1.float()).abs().max()) <= 2 ** -7 * float(dq0.float().abs().max())
    rq, rk, rv = oracle_grads(inp, 1)
    for order in ([2, 0, 3, 1], [3, 2, 1, 0]):
        _, _, (dq, dk, dv) = run_both(w, inp, ring_order=order)
        for g, r in ((dq, rq), (dk, rk), (dv, rv)):
            assert compare(to64(g), r, "bf16").ok


def test_backward_invariants_on_gpu_outputs():
    """sum_j dK_j = 0 and sum_j dV_j = sum_i dO_i per head (every row sees a key)."""
    w, inp = make(128, 2048, 4, 1, None, None, 1, 4)
    _, _, (dq, dk, dv) = run_both(w, inp)
    S = w.S
    tol = 1e-2 * np.sqrt(S)
    np.testing.assert_allclose(to64(dk).sum(axis=1), 0.0, atol=tol)
    np.testing.assert_allclose(to64(dv).sum(axis=1), to64(inp["do"]).sum(axis=1), atol=tol)


def test_fully_masked_rows_have_zero_gradients():
    w, inp = make(128, 256, 1, 1, None, None, 1, 2)
    bias = torch.zeros((1, 256), device=dev())
    bias[0, :3] = float("-inf")
    inp["bias"] = bias
    _, _, (dq, dk, dv) = run_both(w, inp)
    assert torch.all(dq[0, :3] == 0)
    assert torch.all(dk[0, :3] == 0) and torch.all(dv[0, :3] == 0)
    rq, rk, rv = oracle_grads(inp, 1)
    for g, r in ((dq, rq), (dk, rk), (dv, rv)):
        assert compare(to64(g), r, "bf16").ok


def test_autograd_function_matches_explicit_calls():
    w, inp = make(128, 512, 2, 1, None, None, 1, 2)
    q, k, v = (inp[n].clone().requires_grad_(True) for n in ("q", "k", "v"))
    o = ra.RingAttentionFunction.apply(q, k, v, None, None, kw(w))
    o.backward(inp["do"])
    _, _, (dq, dk, dv) = run_both(w, inp)
    assert torch.equal(q.grad, dq) or compare(to64(q.grad), to64(dq), "bf16").ok
    assert torch.equal(k.grad, dk) and torch.equal(v.grad, dv)


def _rows_grad_stored(qh, kh, vh, doh, sub, seg_b=None):
    """dQ rows with Delta from the stored (bf16-rounded) output rows.  ``seg_b``:
    the batch row's segment ids [S] or None."""
    from oracle.attention import _head_backward
    rows = sub[:, 2]
    o_r, lse_r = oracle.attention_rows(qh, kh, vh, sub, None, None if seg_b is None else seg_b[None], 1)
    dq, _, _ = _head_backward(qh[0, rows, 0], kh[0, :, 0], vh[0, :, 0], doh[0, rows, 0],
                              stored(o_r, torch.bfloat16), lse_r, rows, 1, seg_b, None, want_dkdv=False)
    return dq


@pytest.mark.slow
def test_config_causal64k_fwd_bwd():
    """64K causal: dQ on 4096 sampled rows, dK/dV in full on one seeded head, invariants on all heads."""
    w = W.WORKLOADS["causal64k"]
    inp = W.make_inputs(w, dev())
    o, lse, (dq, dk, dv) = run_both(w, inp)
    samples = W.sample_rows(w, None, n=4096)
    rng = np.random.default_rng(w.seed + 5)
    heads = [(0, int(rng.integers(0, w.H)))]
    # dQ rows: oracle per head
    got = to64(dq[torch.as_tensor(samples[:, 0]), torch.as_tensor(samples[:, 2]), torch.as_tensor(samples[:, 1])])
    want = np.zeros_like(got)
    keys = samples[:, 1]
    for h in np.unique(keys):
        idx = np.nonzero(keys == h)[0]
        rows = samples[idx, 2]
        sub = np.stack([np.zeros_like(rows), np.zeros_like(rows), rows], axis=1)
        qh, kh, vh, doh = (to64(inp[n][0, :, int(h)].contiguous())[None, :, None, :] for n in ("q", "k", "v", "do"))
        want[idx] = _rows_grad_stored(qh, kh, vh, doh, sub)
    res = compare(got, want, "bf16")
    assert res.ok, f"dq rows: {res}"
    for b, h in heads:
        qh, kh, vh, doh = (to64(inp[n][b, :, h].contiguous())[None, :, None, :] for n in ("q", "k", "v", "do"))
        o_h, l_h = oracle.attention_forward(qh, kh, vh, None, None, 1)
        _, rk, rv = oracle.attention_backward(qh, kh, vh, doh, None, None, 1, o=stored(o_h, torch.bfloat16), lse=l_h)
        assert compare(to64(dk[b, :, h]), rk[0, :, 0], "bf16").ok
        assert compare(to64(dv[b, :, h]), rv[0, :, 0], "bf16").ok
    tol = 1e-2 * np.sqrt(w.S)
    np.testing.assert_allclose(to64(dk).sum(axis=1), 0.0, atol=tol)
    np.testing.assert_allclose(to64(dv).sum(axis=1), to64(inp["do"]).sum(axis=1), atol=tol)


def _full_size_fwd_bwd(name):
    """A 128K workload at full size, in the bench's launch configuration (B=1,
    H=32, D=128, P=8, chunks 512): O and LSE on 4096 sampled rows, dQ on the
    same rows, dK / dV on 512 sampled keys of one seeded head (including every
    ring-block boundary and, with packed documents, every document start), and
    the invariants on all heads."""
    w = W.WORKLOADS[name]
    inp = W.make_inputs(w, dev(), with_grad_output=True)
    o, lse, (dq, dk, dv) = run_both(w, inp)
    seg = None if inp["seg"] is None else to_np(inp["seg"])
    seg_b = None if seg is None else seg[0]
    samples = W.sample_rows(w, seg, n=4096)
    sel = (torch.as_tensor(samples[:, 0]), torch.as_tensor(samples[:, 2]), torch.as_tensor(samples[:, 1]))
    # forward rows (one head's K / V on the host at a time)
    ro, rl = oracle_rows(inp, samples, 1)
    go, gl = gather_rows(o, lse, samples)
    res = compare(go, ro, "bf16")
    assert res.ok, f"o rows: {res}"
    assert np.abs(gl - rl).max() <= 1e-3
    # dQ rows, Delta from the stored output
    got = to64(dq[sel])
    want = np.zeros_like(got)
    for h in np.unique(samples[:, 1]):
        idx = np.nonzero(samples[:, 1] == h)[0]
        rows = samples[idx, 2]
        sub = np.stack([np.zeros_like(rows), np.zeros_like(rows), rows], axis=1)
        qh, kh, vh, doh = (to64(inp[n][0, :, int(h)].contiguous())[None, :, None, :] for n in ("q", "k", "v", "do"))
        want[idx] = _rows_grad_stored(qh, kh, vh, doh, sub, seg_b)
    res = compare(got, want, "bf16")
    assert res.ok, f"dq rows: {res}"
    # dK / dV on sampled keys of one head (its full forward gives every row's lse and stored o)
    rng = np.random.default_rng(w.seed + 9)
    h = int(rng.integers(0, w.H))
    blk = w.S // w.P
    must = [np.arange(w.P) * blk, np.arange(1, w.P + 1) * blk - 1]
    if seg_b is not None:
        must.append(np.nonzero(np.r_[True, seg_b[1:] != seg_b[:-1]])[0])
    must = np.unique(np.concatenate(must))
    cols = np.unique(np.concatenate([must, rng.choice(w.S, size=512 - len(must), replace=False)]))
    qh, kh, vh, doh = (to64(inp[n][0, :, h].contiguous()) for n in ("q", "k", "v", "do"))
    sg = None if seg is None else seg[:1]
    o_h, l_h = oracle.attention_forward(qh[None, :, None], kh[None, :, None], vh[None, :, None], None, sg, 1)
    rk, rv = oracle.head_backward_cols(qh, kh, vh, doh, stored(o_h, torch.bfloat16)[0, :, 0], l_h[0, 0], cols, 1,
                                       seg_b)
    res = compare(to64(dk[0, torch.as_tensor(cols), h]), rk, "bf16")
    assert res.ok, f"dk cols: {res}"
    res = compare(to64(dv[0, torch.as_tensor(cols), h]), rv, "bf16")
    assert res.ok, f"dv cols: {res}"
    tol = 1e-2 * np.sqrt(w.S)
    sum64 = lambda t: t.double().sum(dim=1).cpu().numpy()    # sums over tokens, in float64 on the device
    np.testing.assert_allclose(sum64(dk), 0.0, atol=tol)
    np.testing.assert_allclose(sum64(dv), sum64(inp["do"]), atol=tol)


@pytest.mark.slow
def test_config_causal128k_fwd_bwd():
    """The bench's workload (128K causal) at full size."""
    _full_size_fwd_bwd("causal128k")


@pytest.mark.slow
def test_config_packed128k_fwd_bwd():
    """128K packed documents (segment masking across documents) at full size, forward and backward."""
    _full_size_fwd_bwd("packed128k")
