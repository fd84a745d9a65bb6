"""The blockwise feed-forward network (ra_feedforward) on the tensor cores.

Compared with the float64 oracle (oracle/feedforward.py) on the same bf16
inputs.  The kernels round the hidden layer h to bf16 between the two
products (relative error at most u = 2^-8 per element), so y may move by up to
u * sum_f |h_f| |W2_of| beyond the bf16 rule's half ulp; the tolerance is
the bf16 rule with that exact bound (checker.operand_rounding_bound), and
the mean bound applies to the excess over half an ulp (y is O(1), so its
own rounding averages ~ulp/4; see checker.py).  Chunk
sizes must not change y at all (rows are independent and every row is
summed in the same order).
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from checker import compare, operand_rounding_bound

pytestmark = pytest.mark.gpu
ra = pytest.importorskip("long_context_exact_ordered_b200")


def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def make(T, dm, dff, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    x = torch.randn((T, dm), generator=g).to(torch.bfloat16)
    w1 = (torch.randn((dff, dm), generator=g) * dm ** -0.5).to(torch.bfloat16)
    w3 = (torch.randn((dff, dm), generator=g) * dm ** -0.5).to(torch.bfloat16)
    w2 = (torch.randn((dm, dff), generator=g) * dff ** -0.5).to(torch.bfloat16)
    return x, w1, w3, w2


CASES = [
    # T, d_model, d_ff, chunk
    (300, 256, 512, 128),       # ragged tokens and chunks
    (1024, 512, 1024, 1024),
    (257, 128, 384, 100),       # d_ff = 3 x 128, d_model below one 256-column output tile
    (2048, 1024, 2816, 512),    # LLaMA-like ratio d_ff = 2.75 d_model
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "T{}-dm{}-dff{}-chunk{}".format(*c))
def test_feedforward_matches_oracle(case):
    T, dm, dff, chunk = case
    x, w1, w3, w2 = make(T, dm, dff, seed=T + dff)
    d = dev()
    y = ra.blockwise_feedforward(x.to(d), w1.to(d), w3.to(d), w2.to(d), chunk_size=chunk)
    torch.cuda.synchronize()
    f64 = lambda t: t.double().numpy()
    ry, h = oracle.blockwise_feedforward(f64(x), f64(w1), f64(w3), f64(w2), chunk_size=chunk, return_hidden=True)
    bound = operand_rounding_bound(np.abs(h) @ np.abs(f64(w2)).T, dff)
    res = compare(y.double().cpu().numpy(), ry, "bf16", rounding_bound=bound, mean_of="excess")
    assert res.ok, str(res)


def test_feedforward_chunking_does_not_change_y():
    x, w1, w3, w2 = make(640, 256, 512, seed=9)
    d = dev()
    args = [t.to(d) for t in (x, w1, w3, w2)]
    base = ra.blockwise_feedforward(*args, chunk_size=640)
    for c in (1, 100, 128, 333):
        assert torch.equal(ra.blockwise_feedforward(*args, chunk_size=c), base)


def test_feedforward_rejects_bad_shapes():
    d = dev()
    x, w1, w3, w2 = (t.to(d) for t in make(64, 128, 256, seed=1))
    with pytest.raises(ra.RingAttnError):
        ra.blockwise_feedforward(x, w1, w3, w2[:, :128].contiguous())
    with pytest.raises(ra.RingAttnError):
        ra.blockwise_feedforward(x.float(), w1.float(), w3.float(), w2.float())
