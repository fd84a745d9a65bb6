"""Pins of the comparison rules in checker.py (CPU only).

The bf16 tolerance rule rests on ``bf16_half_ulp``, and the rule for biased
backward cases on ``oracle.backward_term_magnitudes``.  Both are pinned here
to things other than their own formulas: the bf16 number grid itself (read
from the bit patterns of neighbouring bf16 values), the rounding torch
performs, hand-made planted errors, and closed-form cases in which the
magnitude sums must equal the gradients exactly.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from checker import (BF16_MAX_ABS, BF16_UNIT_ROUNDOFF, bf16_half_ulp, compare, operand_rounding_bound)


def _bf16_neighbours(x):
    """The two bf16 values around |x| (x not itself representable), from bit patterns:
    truncating the fp32 bits toward zero gives the lower one, +1 in the bf16 bit
    pattern the upper one."""
    bits = np.abs(np.asarray(x, dtype=np.float32)).view(np.uint32)
    lo_bits = bits & np.uint32(0xFFFF0000)
    hi_bits = lo_bits + np.uint32(0x10000)
    return lo_bits.view(np.float32).astype(np.float64), hi_bits.view(np.float32).astype(np.float64)


@pytest.mark.parametrize("x", [1e-3, 0.75, 1.0, 3.9, 4.0, 7.99, 100.0, -2.5, 6.1e4])
def test_half_ulp_is_half_the_bf16_spacing(x):
    lo, hi = _bf16_neighbours(np.float32(x))
    assert float(bf16_half_ulp(x)) == (hi - lo) / 2


def test_half_ulp_bounds_torch_rounding_and_is_attained():
    rng = np.random.default_rng(5)
    x = (rng.standard_normal(20000) * np.exp(rng.uniform(-8, 8, 20000))).astype(np.float32)
    rounded = torch.from_numpy(x).to(torch.bfloat16).double().numpy()
    err = np.abs(rounded - x.astype(np.float64))
    assert np.all(err <= bf16_half_ulp(x))
    # a midpoint between two bf16 neighbours rounds by exactly half an ulp
    lo, hi = _bf16_neighbours(np.float32(3.3))
    mid = np.float32((lo + hi) / 2)
    assert abs(float(torch.tensor(mid).to(torch.bfloat16).double()) - float(mid)) == float(bf16_half_ulp(mid))


def test_compare_planted_errors():
    ref = np.concatenate([[0.3, 5.0, -6.0, 100.0], np.linspace(-1, 1, 996)])
    hu = float(bf16_half_ulp(5.0))

    def plant(i, e):
        g = ref.copy()
        g[i] += e
        return g

    assert compare(plant(1, hu + 0.009), ref, "bf16").ok
    assert not compare(plant(1, hu + 0.011), ref, "bf16").ok
    assert not compare(plant(0, 0.0112), ref, "bf16").ok     # half ulp at 0.3 is 2^-10
    # the mean-abs bound applies to the raw error
    assert not compare(ref + 0.0011, ref, "bf16").ok
    # an operand rounding bound above 1e-2 widens only its own element
    bound = np.zeros_like(ref)
    bound[1] = 0.05
    assert compare(plant(1, hu + 0.04), ref, "bf16", rounding_bound=bound).ok
    assert not compare(plant(1, hu + 0.06), ref, "bf16", rounding_bound=bound).ok
    assert not compare(plant(0, 0.04), ref, "bf16", rounding_bound=bound).ok
    # the mean bound on the excess over half an ulp (feed-forward rule): O(1) values
    # rounded to bf16 pass, an added bias of 2e-3 beyond half an ulp does not
    big = np.linspace(1.0, 1.99, 1000)
    rounded = torch.from_numpy(big).to(torch.bfloat16).double().numpy()
    assert not compare(rounded, big, "bf16").ok                       # raw mean ~ ulp/4 > 1e-3
    assert compare(rounded, big, "bf16", mean_of="excess").ok
    assert not compare(big + bf16_half_ulp(big) + 2e-3, big, "bf16", mean_of="excess").ok
    # fp32 rule: raw max-abs
    assert compare(ref + 9e-6, ref, "f32").ok and not compare(plant(2, 1.1e-5), ref, "f32").ok


def test_operand_rounding_bound_value():
    assert operand_rounding_bound(1.0, 0) == BF16_UNIT_ROUNDOFF
    assert operand_rounding_bound(2.0, 1 << 14) == 2.0 * (2.0 ** -8 + 2.0 ** -10)
    assert BF16_MAX_ABS == 1e-2


def _small(seed, S=48, D=8, c=1, seg=False, bias=False):
    rng = np.random.default_rng(seed)
    q, k, v, do = (rng.standard_normal((1, S, 2, D)) for _ in range(4))
    segs = np.repeat(np.arange(3), [S // 3, S // 3, S - 2 * (S // 3)])[None].astype(np.int32) if seg else None
    b = rng.standard_normal((1, S)) if bias else None
    if bias:
        b[0, 5] = -np.inf
    return q, k, v, do, b, segs, c


@pytest.mark.parametrize("seed,c,seg,bias", [(1, 1, False, False), (2, None, True, True), (3, 3, True, False)])
def test_magnitudes_bound_the_gradients(seed, c, seg, bias):
    q, k, v, do, b, segs, c = _small(seed, c=c, seg=seg, bias=bias)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, b, segs, c)
    mq, mk, mv = oracle.backward_term_magnitudes(q, k, v, do, b, segs, c)
    for g, m in ((dq, mq), (dk, mk), (dv, mv)):
        assert np.all(m >= np.abs(g) - 1e-12)
        assert np.all(m >= 0)
    assert float(mq.max()) > 0 and float(mk.max()) > 0


def test_magnitude_of_dv_is_dv_for_nonnegative_upstream_gradient():
    q, k, v, do, b, segs, c = _small(4, seg=True)
    do = np.abs(do)
    _, _, dv = oracle.attention_backward(q, k, v, do, b, segs, c)
    _, _, mv = oracle.backward_term_magnitudes(q, k, v, do, b, segs, c)
    np.testing.assert_allclose(mv, dv, rtol=1e-12, atol=1e-14)


def test_magnitude_of_dq_with_two_opposite_keys():
    """Causal row 1 sees keys 0 and 1, whose dS entries sum to zero; with k_0 = -k_1
    every dQ_1 component is a sum of two terms of equal sign."""
    q, k, v, do, b, segs, c = _small(5)
    k[:, 0] = -k[:, 1]
    dq, _, _ = oracle.attention_backward(q, k, v, do, None, None, 1)
    mq, _, _ = oracle.backward_term_magnitudes(q, k, v, do, None, None, 1)
    np.testing.assert_allclose(mq[0, 1], np.abs(dq[0, 1]), rtol=1e-10)
    assert np.all(mq[0, 0] < 1e-14)         # row 0 sees one key: dS = 0 up to rounding


def test_magnitude_of_dk_for_the_last_causal_key():
    """Under causal masking the last key is seen by the last query only."""
    q, k, v, do, b, segs, c = _small(6)
    _, dk, _ = oracle.attention_backward(q, k, v, do, None, None, 1)
    _, mk, _ = oracle.backward_term_magnitudes(q, k, v, do, None, None, 1)
    np.testing.assert_allclose(mk[0, -1], np.abs(dk[0, -1]), rtol=1e-10)
    assert not np.allclose(mk[0, -2], np.abs(dk[0, -2]))
