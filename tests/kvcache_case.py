"""A shared-prefix serving scenario for the KV-cache tests (CPU and GPU).

One prefix of ``n_prefix`` tokens is cached once (batch 1) and prefilled in
chunks; two requests (batch 2) continue it with their own tokens, appended
and attended chunk by chunk (the last chunk a single decode token).  The
reference for every chunk is the float64 definition of causal attention over
each request's whole sequence (the prefix followed by its own tokens),
evaluated at the chunk's positions.
"""

from __future__ import annotations

import numpy as np
import torch

import oracle


def run_case(make_cache, dtype, device, H, D, n_prefix, prefix_chunks, chunks, seed=71, **attend_kw):
    """Returns a list of (name, got_o, want_o, got_lse, want_lse) per attended chunk."""
    g = torch.Generator().manual_seed(seed)
    S = n_prefix + sum(chunks)
    # per request: q, k, v over its whole sequence; the prefix's k / v are common to both
    q = torch.randn((2, S, H, D), generator=g)
    k = torch.randn((2, S, H, D), generator=g)
    v = torch.randn((2, S, H, D), generator=g)
    k[1, :n_prefix], v[1, :n_prefix], q[1, :n_prefix] = k[0, :n_prefix], v[0, :n_prefix], q[0, :n_prefix]
    q, k, v = (x.to(dtype) for x in (q, k, v))
    ro, rl = oracle.attention_forward(q.double().numpy(), k.double().numpy(), v.double().numpy(), None, None, 1)
    out = []
    prefix = make_cache(1, None)
    pos = 0
    for n in prefix_chunks:                       # prefill of the shared prefix itself
        prefix.append(k[:1, pos:pos + n].to(device), v[:1, pos:pos + n].to(device))
        o, lse = prefix.attend(q[:1, pos:pos + n].to(device), **attend_kw)
        out.append((f"prefix[{pos}:{pos + n}]", o[0], ro[0, pos:pos + n], lse[0], rl[0, :, pos:pos + n]))
        pos += n
    assert pos == n_prefix
    req = make_cache(2, prefix)
    for n in chunks:                              # the two requests' own tokens
        req.append(k[:, pos:pos + n].to(device), v[:, pos:pos + n].to(device))
        o, lse = req.attend(q[:, pos:pos + n].to(device), **attend_kw)
        for b in range(2):
            out.append((f"request {b} [{pos}:{pos + n}]", o[b], ro[b, pos:pos + n], lse[b], rl[b, :, pos:pos + n]))
        pos += n
    return out


def max_errors(results):
    """(max |o error|, max |lse error|) over every chunk (float64 numpy)."""
    eo = el = 0.0
    for _, go, wo, gl, wl in results:
        eo = max(eo, float(np.abs(go.double().cpu().numpy() - wo).max()))
        el = max(el, float(np.abs(gl.double().cpu().numpy() - wl).max()))
    return eo, el
