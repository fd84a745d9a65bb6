"""The oracle's online-softmax step and finalize behind the library's step
signatures (ring_step / finalize), on CPU tensors: lets the tests drive the
host-side ring and cache logic without a GPU."""

from __future__ import annotations

import numpy as np
import torch

import oracle


def oracle_step(q_blk, k_blk, v_blk, q_off, k_off, acc, m, l, bias_blk=None, seg_q=None, seg_k=None,
                 causal_block_size=None):
    B, Sq, H, D = q_blk.shape
    Sk = k_blk.shape[1]
    qpos, kpos = np.arange(q_off, q_off + Sq), np.arange(k_off, k_off + Sk)
    for b in range(B):
        bk = 0 if k_blk.shape[0] == 1 else b        # a key/value block of batch 1 is shared
        for h in range(H):
            st = (m[b, h].double().numpy(), l[b, h].double().numpy(), acc[b, :, h].double().numpy())
            m2, l2, a2 = oracle.online_step(
                st, q_blk[b, :, h].double().numpy(), k_blk[bk, :, h].double().numpy(),
                v_blk[bk, :, h].double().numpy(), qpos, kpos, causal_block_size,
                None if seg_q is None else seg_q[b].numpy(), None if seg_k is None else seg_k[bk].numpy(),
                None if bias_blk is None else bias_blk[bk].double().numpy())
            m[b, h] = torch.from_numpy(m2)
            l[b, h] = torch.from_numpy(l2)
            acc[b, :, h] = torch.from_numpy(a2)


def oracle_finalize(acc, m, l, dtype, out=None, lse=None):
    B, n, H, D = acc.shape
    if out is None:
        out = torch.empty((B, n, H, D), dtype=dtype)
    if lse is None:
        lse = torch.empty((B, H, n), dtype=torch.float32)
    for b in range(B):
        for h in range(H):
            o, ls = oracle.finalize((m[b, h].double().numpy(), l[b, h].double().numpy(), acc[b, :, h].double().numpy()))
            out[b, :, h] = torch.from_numpy(o).to(out.dtype)
            lse[b, h] = torch.from_numpy(ls).float()
    return out, lse
