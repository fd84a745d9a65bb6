"""Comparison rules between a GPU result and the float64 oracle.

Tolerances (stated once, used by every parity test):

* bf16 outputs (fp32 accumulate): max-abs error <= 1e-2 and mean-abs error
  <= 1e-3.  A bf16 output cannot be closer to the exact value than half a
  bf16 ulp, and for |x| >= 4 half an ulp is 0.0156 > 1e-2, so the max-abs
  test is applied to the *excess* over half an ulp of the oracle's value:
  max(0, |gpu - oracle| - ulp_bf16(oracle)/2) <= 1e-2.  The raw max-abs
  error is reported next to it.  The mean-abs bound is applied raw.
* fp32 outputs: max-abs error <= 1e-5 (raw).
* integer outputs (counts, masks): bit-exact.
* bf16 gradients of inputs with a random additive bias: the tensor-core
  backward rounds its product operands dS and P to bf16 (relative error at
  most u = 2^-8 each) before the fp32 sums dQ = scale dS K, dK = scale dS^T Q,
  dV = P^T dO.  Each term then moves by at most u times its magnitude, so a
  correct backward can differ from the exact gradient by up to
  u * sum|terms| (oracle.backward_term_magnitudes), plus the fp32 sums'
  own n * 2^-24 relative error.  When a few keys carry most of the attention
  that bound exceeds 1e-2.  For those cases an element passes when its
  excess over half a bf16 ulp is within max(1e-2, that bound); the mean-abs
  bound stays 1e-3.  Every other case uses the plain bf16 rule.
* the blockwise feed-forward network (no tolerance stated for it): its bf16
  output y is O(1), so rounding it alone averages ~ulp/4 ~ 2e-3; its hidden
  layer is rounded to bf16 between the two products.  Rule: excess over half
  a bf16 ulp within max(1e-2, the hidden layer's rounding bound) per element,
  and the mean of that excess <= 1e-3.
"""

from __future__ import annotations

import dataclasses

import numpy as np

BF16_MAX_ABS = 1e-2
BF16_MEAN_ABS = 1e-3
F32_MAX_ABS = 1e-5
BF16_UNIT_ROUNDOFF = 2.0 ** -8    # round-to-nearest with an 8-bit significand
F32_UNIT_ROUNDOFF = 2.0 ** -24


def operand_rounding_bound(magnitude, n_terms):
    """Largest change of a sum of n_terms products when one factor of every
    term is rounded to bf16 and the sum is formed in fp32: (u_bf16 + n *
    u_f32) * sum|terms|, with ``magnitude`` = sum|terms| element-wise."""
    return (BF16_UNIT_ROUNDOFF + n_terms * F32_UNIT_ROUNDOFF) * np.asarray(magnitude, dtype=np.float64)


def bf16_half_ulp(x):
    """Half the spacing of bf16 numbers at |x| (8 significant bits)."""
    x = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.where(x > 0, x, 1.0)))
    e = np.maximum(e, -126.0)
    return np.where(x > 0, 2.0 ** (e - 8), 2.0 ** -134)


@dataclasses.dataclass
class Cmp:
    ok: bool
    max_abs: float
    mean_abs: float
    max_excess: float
    n: int
    rule: str

    def __str__(self):
        return (f"{self.rule}: ok={self.ok} max_abs={self.max_abs:.3e} "
                f"max_excess={self.max_excess:.3e} mean_abs={self.mean_abs:.3e} n={self.n}")


def compare(gpu, ref, kind="bf16", max_abs=None, mean_abs=None, rounding_bound=None, mean_of="raw") -> Cmp:
    """Compare arrays; ``kind`` is "bf16" (half-ulp excess rule) or "f32".

    ``rounding_bound`` (bf16 only): an array like ``ref`` from
    ``operand_rounding_bound``; the allowed excess of each element is then
    max(max_abs, rounding_bound) instead of max_abs.  ``mean_of`` (bf16
    only): "raw" applies the mean-abs bound to the raw error (the attention
    rule); "excess" applies it to the excess over half a bf16 ulp, for
    outputs with no stated tolerance whose typical magnitude is O(1), where
    the output rounding alone averages about ulp/4 (the feed-forward
    network)."""
    g = np.asarray(gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    both_inf = np.isinf(g) & np.isinf(r) & (np.sign(g) == np.sign(r))
    err = np.where(both_inf, 0.0, np.abs(g - r))
    err = np.where(np.isnan(err), np.inf, err)
    n = err.size
    mx = float(err.max()) if n else 0.0
    mean = float(err.mean()) if n else 0.0
    if kind == "bf16":
        lim = BF16_MAX_ABS if max_abs is None else max_abs
        mlim = BF16_MEAN_ABS if mean_abs is None else mean_abs
        excess = np.maximum(0.0, err - np.where(np.isfinite(r), bf16_half_ulp(r), 0.0))
        if rounding_bound is None:
            allowed = lim
            rule = f"bf16(excess<={lim:g}, mean<={mlim:g})"
        else:
            allowed = np.maximum(lim, np.asarray(rounding_bound, dtype=np.float64))
            rule = f"bf16(excess<=max({lim:g}, operand rounding bound), mean<={mlim:g})"
        over = excess - allowed
        mex = float(excess.max()) if n else 0.0
        if mean_of == "excess":
            mean = float(excess.mean()) if n else 0.0
            rule = rule.replace("mean<=", "mean excess<=")
        ok = (float(over.max()) <= 0.0 if n else True) and mean <= mlim
    else:
        lim = F32_MAX_ABS if max_abs is None else max_abs
        mex = mx
        ok = mx <= lim and (mean_abs is None or mean <= mean_abs)
        rule = f"f32(max<={lim:g})"
    return Cmp(ok, mx, mean, mex, n, rule)
