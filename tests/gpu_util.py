"""Helpers shared by the GPU parity tests: device->host copies for the oracle."""

from __future__ import annotations

import numpy as np
import torch

import oracle


def to64(t):
    return None if t is None else t.detach().float().cpu().double().numpy()


def to_np(t):
    return None if t is None else t.detach().cpu().numpy()


def oracle_full(inp, c):
    """Oracle forward over the whole problem (small sizes)."""
    return oracle.attention_forward(to64(inp["q"]), to64(inp["k"]), to64(inp["v"]), to64(inp.get("bias")),
                                    to_np(inp.get("seg")), c)


def oracle_rows(inp, samples, c):
    """Oracle forward for sampled (b, h, i) rows, one head's K/V on the host at a time."""
    q, k, v = inp["q"], inp["k"], inp["v"]
    bias, seg = inp.get("bias"), inp.get("seg")
    D = q.shape[-1]
    o = np.zeros((len(samples), D))
    lse = np.zeros(len(samples))
    keys = samples[:, 0] * (1 << 20) + samples[:, 1]
    for key in np.unique(keys):
        idx = np.nonzero(keys == key)[0]
        b, h = int(samples[idx[0], 0]), int(samples[idx[0], 1])
        rows = samples[idx, 2]
        kh = to64(k[b, :, h].contiguous())[None, :, None, :]
        vh = to64(v[b, :, h].contiguous())[None, :, None, :]
        qr = to64(q[b, torch.as_tensor(rows, device=q.device), h])
        sub = np.stack([np.zeros_like(rows), np.zeros_like(rows), rows], axis=1)
        o[idx], lse[idx] = oracle.attention_rows(None, kh, vh, sub, None if bias is None else to64(bias[b:b + 1]),
                                                 None if seg is None else to_np(seg[b:b + 1]), c, q_rows=qr)
    return o, lse


def gather_rows(o, lse, samples):
    """GPU outputs at sampled (b, h, i) rows -> numpy float64."""
    s = torch.as_tensor(samples, device=o.device)
    return to64(o[s[:, 0], s[:, 2], s[:, 1]]), to64(lse[s[:, 0], s[:, 1], s[:, 2]])
