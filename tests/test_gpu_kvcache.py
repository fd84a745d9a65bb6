"""KV-cache ring steps on the tensor cores (needs a B200).

A shared prefix cached once (batch 1) serves two requests through ra_step's
shared key/value side; prefill chunks and a single-token decode step are
checked against the float64 definition of causal attention over each
request's whole sequence: bf16 under the bf16 rule of checker.py, fp32 (the
CUDA-core step) at 1e-5.  LSE within 1e-3 (bf16) / 1e-5 (fp32).
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

from checker import compare
from kvcache_case import run_case

pytestmark = pytest.mark.gpu
ra = pytest.importorskip("long_context_exact_ordered_b200")
from long_context_exact_ordered_b200.kvcache import KVCache  # noqa: E402


def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


@pytest.mark.parametrize("dtype,block,D", [(torch.bfloat16, 256, 128), (torch.bfloat16, 384, 64),
                                           (torch.float32, 256, 64)])
def test_kvcache_prefix_sharing_prefill_and_decode(dtype, block, D):
    H = 4
    d = dev()

    def make(batch, prefix):
        return KVCache(batch, H, D, capacity=2048, block=block, dtype=dtype, device=d, prefix=prefix)

    res = run_case(make, dtype, d, H, D, n_prefix=1000, prefix_chunks=(512, 488), chunks=(300, 399, 1))
    torch.cuda.synchronize()
    assert ra.device_status() == 0
    kind, lse_tol = ("bf16", 1e-3) if dtype == torch.bfloat16 else ("f32", 1e-5)
    for name, go, wo, gl, wl in res:
        r = compare(go.double().cpu().numpy(), wo, kind)
        assert r.ok, f"{name}: {r}"
        assert float(np.abs(gl.double().cpu().numpy() - wl).max()) <= lse_tol, name
