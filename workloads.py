"""Seeded synthetic inputs for Ring Attention workloads.

This module only draws inputs: shapes, random tensors, packed-document
segment ids and the rows sampled for checking.  It holds none of the
attention arithmetic, so both the CUDA path's tests/bench and the CPU oracle
can take their inputs from it without sharing any computation.

Workloads (sizes of the pages' long-context setting: sequences cut into P
ring blocks, query/key chunks of 512, causal_block_size 1 for causal):

=============  ==  ==  ===  =========  =  =====  ======  ========================
name           B   H   D    S          P  chunk  causal  inputs
=============  ==  ==  ===  =========  =  =====  ======  ========================
tiny           1   2   64   1024       4  128    1       fp32 N(0,1), forward
noncausal32k   2   16  64   32768      8  512    no      bf16 N(0,1), bias = 0
packed128k     1   32  128  131072     8  512    1       bf16 N(0,1), packed docs
causal128k     1   32  128  131072     8  512    1       bf16 N(0,1) (+dO)
causal64k      1   32  128  65536      8  512    1       bf16 N(0,1) + dO, fwd+bwd
causal1m       1   32  128  1048576    8  512    1       bf16 N(0,1)/sqrt(128)
causal16k      1   32  128  16384      8  512    1       bf16 N(0,1) + dO (profiling)
causal32k      1   32  128  32768      8  512    1       bf16 N(0,1) + dO (profiling)
causal128k_c64 1  32  128  131072     8  512    64      bf16 N(0,1) + dO, block-causal
causal128k_c512 1 32  128  131072     8  512    512     bf16 N(0,1) + dO, block-causal
=============  ==  ==  ===  =========  =  =====  ======  ========================

Random tensors: ``torch.Generator(device).manual_seed(seed)``, drawn in the
fixed order q, k, v, dO, each ``randn`` in fp32 (times the stated scale),
then cast to the working dtype with round-to-nearest-even.  Packed documents:
lengths drawn uniformly (inclusive) from [1024, 32768] with
``numpy.random.default_rng(seed + 11)`` until they cover S, the last one
truncated; segment id = document index.
"""

from __future__ import annotations

import dataclasses

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    D: int
    S: int
    P: int
    chunk: int
    causal_block_size: int | None
    dtype: str = "bf16"             # "bf16" or "f32"
    segments: str | None = None     # None or "packed"
    bias: str | None = None         # None, "zeros"
    backward: bool = False
    seed: int = 0
    std: float = 1.0
    description: str = ""
    doc_lo: int = 1024              # packed-document length range (inclusive)
    doc_hi: int = 32768


WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny", 1, 2, 64, 1024, 4, 128, 1, dtype="f32", seed=1001,
                 description="tiny causal ring attention, fp32, forward"),
        Workload("noncausal32k", 2, 16, 64, 32768, 8, 512, None, bias="zeros", seed=1002,
                 description="non-causal forward, d_model 1024, attention_bias = 0"),
        Workload("packed128k", 1, 32, 128, 131072, 8, 512, 1, segments="packed", seed=1003,
                 description="causal packed-document forward, segment masking"),
        Workload("causal128k", 1, 32, 128, 131072, 8, 512, 1, backward=True, seed=1003,
                 description="causal forward+backward at 128K tokens"),
        Workload("causal64k", 1, 32, 128, 65536, 8, 512, 1, backward=True, seed=1004,
                 description="causal forward+backward with saved LSE"),
        Workload("causal1m", 1, 32, 128, 1048576, 8, 512, 1, seed=1005, std=128 ** -0.5,
                 description="million-token causal forward"),
        Workload("causal16k", 1, 32, 128, 16384, 8, 512, 1, backward=True, seed=1006,
                 description="profiling size: causal forward+backward, every input larger than L2"),
        Workload("causal32k", 1, 32, 128, 32768, 8, 512, 1, backward=True, seed=1007,
                 description="profiling size: causal forward+backward, second point of DRAM scaling"),
        Workload("causal128k_c64", 1, 32, 128, 131072, 8, 512, 64, backward=True, seed=1003,
                 description="block-causal (causal_block_size 64) forward+backward at 128K tokens"),
        Workload("causal128k_c512", 1, 32, 128, 131072, 8, 512, 512, backward=True, seed=1003,
                 description="block-causal (causal_block_size 512) forward+backward at 128K tokens"),
    ]
}


def packed_segment_ids(S: int, seed: int, lo: int = 1024, hi: int = 32768) -> np.ndarray:
    """Segment ids of packed documents covering S tokens (int32 [S])."""
    rng = np.random.default_rng(seed + 11)
    lengths = []
    total = 0
    while total < S:
        n = int(rng.integers(lo, hi, endpoint=True))
        n = min(n, S - total)
        lengths.append(n)
        total += n
    return np.repeat(np.arange(len(lengths), dtype=np.int32), lengths)


def make_inputs(w: Workload, device="cpu", with_grad_output: bool | None = None, seed: int | None = None):
    """Draw the workload's tensors on ``device``.

    Returns a dict with q, k, v (and do when the workload has a backward or
    ``with_grad_output``), plus ``bias`` (fp32 [B,S] or None) and ``seg``
    (int32 [B,S] or None), all torch tensors on ``device``.
    """
    import torch

    seed = w.seed if seed is None else seed
    want_do = w.backward if with_grad_output is None else with_grad_output
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    shape = (w.B, w.S, w.H, w.D)
    out = {}
    names = ["q", "k", "v"] + (["do"] if want_do else [])
    for name in names:
        x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
        if w.std != 1.0:
            x.mul_(w.std)
        out[name] = x.to(dt)
        del x
    out["bias"] = torch.zeros((w.B, w.S), device=device, dtype=torch.float32) if w.bias == "zeros" else None
    if w.segments == "packed":
        seg = torch.from_numpy(packed_segment_ids(w.S, seed, w.doc_lo, w.doc_hi)).to(device)
        out["seg"] = seg.unsqueeze(0).expand(w.B, w.S).contiguous()
    else:
        out["seg"] = None
    return out


def sample_rows(w: Workload, seg=None, n: int = 4096, seed: int | None = None) -> np.ndarray:
    """Distinct (b, h, i) rows to check, int64 [n, 3].

    Always includes rows 0 and S-1, the first and last row of every ring
    block and the first row of every segment (spread over heads
    round-robin); the rest are uniform from ``default_rng(seed + 7)``.
    """
    seed = w.seed if seed is None else seed
    rng = np.random.default_rng(seed + 7)
    blk = w.S // w.P
    must = {0, w.S - 1}
    for r in range(w.P):
        must.add(r * blk)
        must.add((r + 1) * blk - 1)
    if seg is not None:
        s0 = np.asarray(seg)[0]
        starts = np.nonzero(np.r_[True, s0[1:] != s0[:-1]])[0]
        must.update(int(x) for x in starts)
    chosen = set()
    out = []
    for t, i in enumerate(sorted(must)):
        key = (t % w.B, (t * 7) % w.H, i)
        chosen.add(key)
        out.append(key)
    total = w.B * w.H * w.S
    n = min(n, total)
    while len(out) < n:
        flat = rng.integers(0, total, size=2 * (n - len(out)) + 16)
        for f in flat:
            key = (int(f // (w.H * w.S)), int((f // w.S) % w.H), int(f % w.S))
            if key not in chosen:
                chosen.add(key)
                out.append(key)
                if len(out) == n:
                    break
    return np.asarray(out, dtype=np.int64)


def small_workload(B=1, H=2, D=64, S=512, P=2, chunk=128, causal_block_size=1, dtype="bf16",
                   segments=None, bias=None, seed=7, std=1.0, backward=False,
                   doc_lo=1024, doc_hi=32768) -> Workload:
    """An ad-hoc workload for parity tests at sizes the oracle finishes in seconds."""
    return Workload(f"small_B{B}H{H}D{D}S{S}P{P}", B, H, D, S, P, chunk, causal_block_size, dtype=dtype,
                    segments=segments, bias=bias, backward=backward, seed=seed, std=std,
                    doc_lo=doc_lo, doc_hi=doc_hi)
