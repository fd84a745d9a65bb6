"""Pins of the CPU oracle to facts outside itself (no GPU).

Each test ties the oracle to something the pages or the mathematics fix:
brute-force loops, a library routine (torch's float64 SDPA), the ring route,
closed forms, invariances, finite differences, a worked ring schedule from the
pages' send/receive rule, and a negative control.  A plausible mistake in the
oracle (a dropped bias, a flipped causal compare, a transposed operand, a
wrong scale) fails at least one of them; ``test_planted_mistakes`` checks that
claim by planting such mistakes in a copy of the oracle's arithmetic.
"""

from __future__ import annotations

import itertools
import math
import os

import numpy as np
import pytest

import oracle
from oracle import loops
from oracle.attention import attention_backward_rows
from checker import compare
from negative_control import boundary_window_attention

RNG = np.random.default_rng(12345)
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand(*shape, rng=RNG, scale=1.0):
    return rng.standard_normal(shape) * scale


def tiny_case(S=16, D=8, B=1, H=1, seg=False, bias=False, neg_inf_bias=False, rng=RNG):
    q, k, v, do = (rand(B, S, H, D, rng=rng) for _ in range(4))
    segs = None
    if seg:
        cuts = sorted(rng.choice(np.arange(1, S), size=2, replace=False))
        segs = np.zeros((B, S), dtype=np.int32)
        segs[:, cuts[0]:] += 1
        segs[:, cuts[1]:] += 1
    bs = None
    if bias:
        bs = rand(B, S, rng=rng)
        if neg_inf_bias:
            bs[:, 0] = -np.inf      # masks key 0: causal row 0 then has no visible key
            bs[:, S // 2] = -np.inf
    return q, k, v, do, segs, bs


# --------------------------------------------------------------------------- P1

MASKS = [
    dict(c=None, seg=False, bias=False),
    dict(c=1, seg=False, bias=False),
    dict(c=3, seg=False, bias=False),
    dict(c=1, seg=True, bias=False),
    dict(c=None, seg=True, bias=True),
    dict(c=1, seg=True, bias=True, neg_inf_bias=True),
    dict(c=2, seg=False, bias=True, neg_inf_bias=True),
]


@pytest.mark.parametrize("mask", MASKS, ids=lambda m: "-".join(f"{k}{v}" for k, v in m.items()))
@pytest.mark.parametrize("S,D", [(13, 4), (24, 8)])
def test_forward_matches_python_loops(mask, S, D):
    q, k, v, do, seg, bias = tiny_case(S, D, seg=mask["seg"], bias=mask["bias"],
                                       neg_inf_bias=mask.get("neg_inf_bias", False))
    o, lse = oracle.attention_forward(q, k, v, bias, seg, mask["c"])
    ol, ll = loops.forward_loops(q[0, :, 0].tolist(), k[0, :, 0].tolist(), v[0, :, 0].tolist(),
                                 None if bias is None else bias[0].tolist(),
                                 None if seg is None else seg[0].tolist(), mask["c"])
    np.testing.assert_allclose(o[0, :, 0], np.array(ol), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse[0, 0], np.array(ll), rtol=0, atol=1e-12)


@pytest.mark.parametrize("mask", MASKS[:4] + MASKS[5:], ids=lambda m: "-".join(f"{k}{v}" for k, v in m.items()))
def test_backward_matches_python_loops(mask):
    S, D = 12, 4
    q, k, v, do, seg, bias = tiny_case(S, D, seg=mask["seg"], bias=mask["bias"],
                                       neg_inf_bias=mask.get("neg_inf_bias", False))
    dq, dk, dv = oracle.attention_backward(q, k, v, do, bias, seg, mask["c"])
    lq, lk, lv = loops.backward_loops(q[0, :, 0].tolist(), k[0, :, 0].tolist(), v[0, :, 0].tolist(),
                                      do[0, :, 0].tolist(), None if bias is None else bias[0].tolist(),
                                      None if seg is None else seg[0].tolist(), mask["c"])
    for a, b in ((dq, lq), (dk, lk), (dv, lv)):
        np.testing.assert_allclose(a[0, :, 0], np.array(b), rtol=0, atol=1e-11)


@pytest.mark.parametrize("c", [None, 1, 4])
def test_forward_matches_torch_sdpa_float64(c):
    """A library routine: torch's scaled_dot_product_attention on CPU in float64."""
    torch = pytest.importorskip("torch")
    B, S, H, D = 2, 48, 3, 16
    q, k, v, do, seg, bias = tiny_case(S, D, B=B, H=H, seg=True, bias=True)
    o, lse = oracle.attention_forward(q, k, v, bias, seg, c)
    for b in range(B):
        vis = oracle.visible_mask(np.arange(S), S, c, seg[b], bias[b])
        am = torch.from_numpy(np.where(vis, bias[b][None, :], -np.inf))
        qt = torch.from_numpy(q[b].transpose(1, 0, 2).copy())
        kt = torch.from_numpy(k[b].transpose(1, 0, 2).copy())
        vt = torch.from_numpy(v[b].transpose(1, 0, 2).copy())
        ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=am).numpy()
        np.testing.assert_allclose(o[b].transpose(1, 0, 2), ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("P", [1, 2, 4, 8])
@pytest.mark.parametrize("mask", [MASKS[0], MASKS[1], MASKS[3], MASKS[5]],
                         ids=lambda m: "-".join(f"{k}{v}" for k, v in m.items()))
def test_ring_blockwise_equals_definition(P, mask):
    S, D = 64, 8
    q, k, v, do, seg, bias = tiny_case(S, D, B=2, H=2, seg=mask["seg"], bias=mask["bias"],
                                       neg_inf_bias=mask.get("neg_inf_bias", False))
    o, lse = oracle.attention_forward(q, k, v, bias, seg, mask["c"])
    blk = S // P
    for qc, kc in [(blk, blk), (max(1, blk // 2), max(1, blk // 4))]:
        for merge in ("online", "lse"):
            ro, rl = oracle.ring_blockwise_reference(q, k, v, bias, seg, mask["c"], P, qc, kc, merge=merge)
            np.testing.assert_allclose(ro, o, rtol=0, atol=1e-12)
            np.testing.assert_allclose(rl, lse, rtol=0, atol=1e-12)


def test_attention_rows_matches_full():
    S, D = 40, 8
    q, k, v, do, seg, bias = tiny_case(S, D, B=2, H=3, seg=True, bias=True, neg_inf_bias=True)
    o, lse = oracle.attention_forward(q, k, v, bias, seg, 1)
    samples = np.array([(b, h, i) for b in range(2) for h in range(3) for i in range(0, S, 3)])
    ro, rl = oracle.attention_rows(q, k, v, samples, bias, seg, 1)
    np.testing.assert_allclose(ro, o[samples[:, 0], samples[:, 2], samples[:, 1]], atol=1e-13)
    np.testing.assert_allclose(rl, lse[samples[:, 0], samples[:, 1], samples[:, 2]], atol=1e-13)
    dq, _, _ = oracle.attention_backward(q, k, v, do, bias, seg, 1)
    rdq = attention_backward_rows(q, k, v, do, samples, bias, seg, 1)
    np.testing.assert_allclose(rdq, dq[samples[:, 0], samples[:, 2], samples[:, 1]], atol=1e-12)


# --------------------------------------------------------------------------- P2 / P3

@pytest.mark.parametrize("P", [2, 3, 4])
def test_ring_order_invariance_all_permutations(P):
    S, D = 12 * P, 8
    q, k, v, do, seg, bias = tiny_case(S, D, seg=True, bias=True)
    base, bl = oracle.ring_blockwise_reference(q, k, v, bias, seg, 1, P)
    for perm in itertools.permutations(range(P)):
        o, l = oracle.ring_blockwise_reference(q, k, v, bias, seg, 1, P, order=perm)
        np.testing.assert_allclose(o, base, atol=1e-12)
        np.testing.assert_allclose(l, bl, atol=1e-12)


def test_ring_order_invariance_p8_random():
    P, S, D = 8, 64, 8
    q, k, v, do, seg, bias = tiny_case(S, D, H=2)
    base, bl = oracle.ring_blockwise_reference(q, k, v, None, None, None, P)
    rng = np.random.default_rng(3)
    for _ in range(6):
        perm = rng.permutation(P)
        for merge in ("online", "lse"):
            o, l = oracle.ring_blockwise_reference(q, k, v, None, None, None, P, order=perm, merge=merge)
            np.testing.assert_allclose(o, base, atol=1e-12)
            np.testing.assert_allclose(l, bl, atol=1e-12)


def test_chunk_size_invariance():
    P, S, D = 2, 64, 8
    q, k, v, do, seg, bias = tiny_case(S, D, seg=True)
    base, bl = oracle.attention_forward(q, k, v, None, seg, 1)
    for qc in (1, 2, 4, 8, 16, 32):
        for kc in (1, 4, 16, 32):
            o, l = oracle.ring_blockwise_reference(q, k, v, None, seg, 1, P, qc, kc)
            np.testing.assert_allclose(o, base, atol=1e-12)
            np.testing.assert_allclose(l, bl, atol=1e-12)


def test_lse_merge_is_order_free_and_exact():
    n, D = 7, 5
    parts = []
    for t in range(4):
        o = rand(n, D)
        l = rand(n)
        l[t] = -np.inf           # some empty partials
        o[t] = 0.0
        parts.append((o, l))
    exact_l = np.log(sum(np.exp(p[1]) for p in parts))
    exact_o = sum(np.exp(p[1] - exact_l)[:, None] * p[0] for p in parts)
    for perm in itertools.permutations(range(4)):
        mo, ml = np.zeros((n, D)), np.full(n, -np.inf)
        for i in perm:
            mo, ml = oracle.lse_merge(mo, ml, *parts[i])
        np.testing.assert_allclose(ml, exact_l, atol=1e-13)
        np.testing.assert_allclose(mo, exact_o, atol=1e-13)
    eo, el = oracle.lse_merge(np.zeros((1, D)), np.array([-np.inf]), np.zeros((1, D)), np.array([-np.inf]))
    assert el[0] == -np.inf and np.all(eo == 0)


# --------------------------------------------------------------------------- P4 / P5 / P6

@pytest.mark.parametrize("c", [None, 1, 5])
def test_zero_queries_give_mean_of_visible_values(c):
    S, D = 30, 6
    q, k, v, do, seg, bias = tiny_case(S, D, B=2, H=2, seg=True)
    q[:] = 0.0
    o, lse = oracle.attention_forward(q, k, v, None, seg, c)
    for b in range(2):
        vis = oracle.visible_mask(np.arange(S), S, c, seg[b])
        n = vis.sum(axis=1)
        for h in range(2):
            mean = (vis.astype(float) @ v[b, :, h]) / n[:, None]
            np.testing.assert_allclose(o[b, :, h], mean, atol=1e-13)
            np.testing.assert_allclose(lse[b, h], np.log(n), atol=1e-13)


def test_softmax_rows_sum_to_one_and_single_key_rows():
    S, D = 32, 8
    q, k, v, do, seg, bias = tiny_case(S, D, seg=True, bias=True)
    o, lse = oracle.attention_forward(q, k, v, bias, seg, 1)
    scale = 1 / math.sqrt(D)
    vis = oracle.visible_mask(np.arange(S), S, 1, seg[0], bias[0])
    s = scale * q[0, :, 0] @ k[0, :, 0].T + bias[0][None, :]
    p = np.where(vis, np.exp(s - lse[0, 0][:, None]), 0.0)
    np.testing.assert_allclose(p.sum(axis=1), 1.0, atol=1e-13)
    # causal row 0 and every segment's first row see exactly one key: o = v of that key
    starts = np.nonzero(np.r_[True, seg[0][1:] != seg[0][:-1]])[0]
    for i in starts:
        np.testing.assert_array_equal(o[0, i, 0], v[0, i, 0])


def test_shift_invariance():
    S, D = 24, 8
    q, k, v, do, seg, bias = tiny_case(S, D, seg=True, bias=True)
    o, lse = oracle.attention_forward(q, k, v, bias, seg, 1)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, bias, seg, 1)
    cvec = rand(D)
    o2, lse2 = oracle.attention_forward(q, k + cvec, v, bias, seg, 1)
    np.testing.assert_allclose(o2, o, atol=1e-10)
    np.testing.assert_allclose(lse2[0, 0] - lse[0, 0], q[0, :, 0] @ cvec / math.sqrt(D), atol=1e-10)
    dq2, _, _ = oracle.attention_backward(q, k + cvec, v, do, bias, seg, 1)
    np.testing.assert_allclose(dq2, dq, atol=1e-10)
    o3, lse3 = oracle.attention_forward(q, k, v, bias + 2.5, seg, 1)
    np.testing.assert_allclose(o3, o, atol=1e-10)
    np.testing.assert_allclose(lse3, lse + 2.5, atol=1e-10)
    dq3, dk3, dv3 = oracle.attention_backward(q, k, v, do, bias + 2.5, seg, 1)
    for a, b in ((dq3, dq), (dk3, dk), (dv3, dv)):
        np.testing.assert_allclose(a, b, atol=1e-10)


def test_fully_masked_rows():
    S, D = 10, 4
    q, k, v, do, seg, bias = tiny_case(S, D, bias=True, neg_inf_bias=True)
    o, lse = oracle.attention_forward(q, k, v, bias, None, 1)
    assert lse[0, 0, 0] == -np.inf and np.all(o[0, 0, 0] == 0)      # row 0 sees only key 0 (masked)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, bias, None, 1)
    assert np.all(dq[0, 0, 0] == 0)
    assert np.all(dk[0, 0, 0] == 0) and np.all(dv[0, 0, 0] == 0)     # a masked key gets no gradient


# --------------------------------------------------------------------------- P7

def test_visible_counts_closed_forms():
    S = 200
    rows = np.arange(S)
    np.testing.assert_array_equal(oracle.visible_count_rows(rows, S, None), np.full(S, S))
    np.testing.assert_array_equal(oracle.visible_count_rows(rows, S, 1), rows + 1)
    for c in (2, 7, 64):
        np.testing.assert_array_equal(oracle.visible_count_rows(rows, S, c),
                                      np.minimum(S, (rows // c + 1) * c))
    lengths = [37, 80, 1, 82]
    seg = np.repeat(np.arange(4), lengths)
    start = np.repeat(np.cumsum([0] + lengths[:-1]), lengths)
    np.testing.assert_array_equal(oracle.visible_count_rows(rows, S, 1, seg), rows - start + 1)
    assert oracle.visible_pairs_total(2, 3, S, 1) == 2 * 3 * S * (S + 1) // 2
    assert oracle.visible_pairs_total(1, 1, S, 1, seg[None]) == sum(L * (L + 1) // 2 for L in lengths)
    assert oracle.visible_pairs_total(1, 2, S, None) == 2 * S * S


def test_visible_column_counts_closed_forms():
    """Per key j: the number of query rows that see it (what the backward's
    debug counter is compared with), from closed forms, not from the mask."""
    S = 200
    j = np.arange(S)
    np.testing.assert_array_equal(oracle.visible_count_cols(S, None), np.full(S, S))
    np.testing.assert_array_equal(oracle.visible_count_cols(S, 1), S - j)
    for c in (2, 7, 64):
        # queries i with i // c >= j // c are i >= (j // c) * c
        np.testing.assert_array_equal(oracle.visible_count_cols(S, c), S - (j // c) * c)
    lengths = [37, 80, 1, 82]
    seg = np.repeat(np.arange(4), lengths)
    end = np.repeat(np.cumsum(lengths), lengths)                  # exclusive end of j's document
    np.testing.assert_array_equal(oracle.visible_count_cols(S, 1, seg), end - j)
    np.testing.assert_array_equal(oracle.visible_count_cols(S, None, seg), np.repeat(lengths, lengths))
    bias = np.zeros(S)
    bias[[0, 5, 199]] = -np.inf
    want = (S - j).astype(np.int64)
    want[[0, 5, 199]] = 0                                         # a -inf bias masks the key for everyone
    np.testing.assert_array_equal(oracle.visible_count_cols(S, 1, None, bias), want)
    # rows and columns count the same pairs
    for c, sg, bs in ((1, seg, None), (3, None, bias), (None, seg, bias)):
        assert oracle.visible_count_cols(S, c, sg, bs).sum() == oracle.visible_count_rows(j, S, c, sg, bs).sum()


# --------------------------------------------------------------------------- P8 / P9

def test_backward_matches_finite_differences():
    S, D = 9, 3
    q, k, v, do, seg, bias = tiny_case(S, D, seg=True, bias=True)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, bias, seg, 2)

    def loss(qq, kk, vv):
        o, _ = oracle.attention_forward(qq, kk, vv, bias, seg, 2)
        return float(np.sum(do * o))

    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp = x.copy(); xp[idx] += h
            xm = x.copy(); xm[idx] -= h
            args_p = {"q": (xp, k, v), "k": (q, xp, v), "v": (q, k, xp)}[name]
            args_m = {"q": (xm, k, v), "k": (q, xm, v), "v": (q, k, xm)}[name]
            num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        np.testing.assert_allclose(g, num, rtol=1e-6, atol=1e-8, err_msg=name)


def test_backward_on_sampled_keys_equals_full_backward():
    """head_backward_cols (dK, dV at chosen keys) against the full backward,
    itself pinned by finite differences above."""
    S, D = 70, 8
    q, k, v, do, seg, bias = tiny_case(S, D, seg=True, bias=True, neg_inf_bias=True)
    c = 3
    o, lse = oracle.attention_forward(q, k, v, bias, seg, c)
    _, dk, dv = oracle.attention_backward(q, k, v, do, bias, seg, c, o=o, lse=lse)
    cols = np.array([0, 1, 5, 33, 34, 69])
    f = lambda x: np.asarray(x, dtype=np.float64)[0, :, 0]
    gk, gv = oracle.head_backward_cols(f(q), f(k), f(v), f(do), f(o), np.asarray(lse)[0, 0], cols, c,
                                       np.asarray(seg)[0], np.asarray(bias, dtype=np.float64)[0])
    np.testing.assert_allclose(gk, dk[0, cols, 0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(gv, dv[0, cols, 0], rtol=0, atol=1e-12)


def test_backward_invariants():
    S, D = 40, 8
    q, k, v, do, seg, bias = tiny_case(S, D, B=2, H=2, seg=True)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, None, seg, 1)
    np.testing.assert_allclose(dk.sum(axis=1), 0.0, atol=1e-12)          # sum_j dS_ij = 0
    np.testing.assert_allclose(dv.sum(axis=1), do.sum(axis=1), atol=1e-12)  # every row sees a key


# --------------------------------------------------------------------------- ring schedule

def test_ring_schedule_matches_send_receive_rule():
    """Simulate send-to-next / receive-from-previous and check the golden table."""
    rows = [list(map(int, ln.split())) for ln in open(os.path.join(GOLDEN, "ring_schedule_p4.txt"))
            if ln.strip() and not ln.startswith("#")]
    P = 4
    held = list(range(P))                    # rank r starts with block r
    for t in range(P):
        assert rows[t] == [t] + held
        assert held == [(r - t) % P for r in range(P)]
        held = [held[(r - 1) % P] for r in range(P)]   # receive the previous rank's block


# --------------------------------------------------------------------------- P10

def test_negative_control_boundary_window_fails_checker():
    rng = np.random.default_rng(5)
    B, S, H, D, P = 1, 256, 2, 16, 4
    q, k, v = (rng.standard_normal((B, S, H, D)) for _ in range(3))
    exact, _ = oracle.attention_forward(q, k, v, None, None, 1)
    approx = boundary_window_attention(q, k, v, P, overlap=8)
    res = compare(approx, exact, "bf16")
    assert not res.ok and res.max_abs > 1e-2, str(res)
    # ...while the exact ring route passes the same checker
    ring, _ = oracle.ring_blockwise_reference(q, k, v, None, None, 1, P, 16, 16)
    assert compare(ring, exact, "bf16").ok


# --------------------------------------------------------------------------- planted mistakes

def _planted_forward(q, k, v, bias, seg, c, mistake):
    """A copy of the definition with one deliberate mistake (CPU only)."""
    B, S, H, D = q.shape
    scale = 1 / math.sqrt(D) if mistake != "scale" else 1 / D
    o = np.zeros_like(q)
    for b in range(B):
        for h in range(H):
            s = scale * (q[b, :, h] @ (k[b, :, h].T if mistake != "transpose" else k[b, :, h][::-1].T))
            if bias is not None and mistake != "drop_bias":
                s = s + bias[b][None, :]
            i = np.arange(S)[:, None]
            j = np.arange(S)[None, :]
            vis = (i >= j) if mistake != "flip_causal" else (i + 1 >= j)   # off by one: sees the next key
            if seg is not None:
                vis = vis & (seg[b][:, None] == seg[b][None, :])
            s = np.where(vis, s, -np.inf)
            e = np.exp(s - s.max(axis=1, keepdims=True))
            o[b, :, h] = (e @ v[b, :, h]) / e.sum(axis=1, keepdims=True)
    return o


@pytest.mark.parametrize("mistake", ["scale", "transpose", "drop_bias", "flip_causal"])
def test_planted_mistakes_are_caught(mistake):
    S, D = 24, 8
    q, k, v, do, seg, bias = tiny_case(S, D, seg=True, bias=True)
    ok = _planted_forward(q, k, v, bias, seg, 1, "none")
    ref, _ = loops.forward_loops(q[0, :, 0].tolist(), k[0, :, 0].tolist(), v[0, :, 0].tolist(),
                                 bias[0].tolist(), seg[0].tolist(), 1)
    np.testing.assert_allclose(ok[0, :, 0], np.array(ref), atol=1e-12)
    bad = _planted_forward(q, k, v, bias, seg, 1, mistake)
    assert np.max(np.abs(bad[0, :, 0] - np.array(ref))) > 1e-3
