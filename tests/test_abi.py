"""The C ABI library: loads without a GPU, exports every declared symbol, and
rejects bad arguments on the host before any device work (no GPU needed)."""

from __future__ import annotations

import ctypes
import os
import re

import numpy as np
import pytest

from long_context_exact_ordered_b200 import _lib
from long_context_exact_ordered_b200 import api
import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ringattn.h")
DEBUG_HEADER = os.path.join(ROOT, "include", "ringattn_debug.h")


def declared_functions(header=HEADER):
    text = open(header).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ra_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported():
    lib = _lib.load()
    names = declared_functions()
    assert {"ra_forward", "ra_backward", "ra_step", "ra_finalize", "ra_lse_merge", "ra_workspace_size",
            "ra_get_device_status", "ra_strerror", "ra_count_visible_pairs", "ra_ring_schedule"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n
        assert n in _lib.SIGNATURES, n


def test_debug_build_exports_its_extra_symbol():
    """The RA_DEBUG_COUNT build exports everything both headers declare; the
    release build does not carry the debug entry point."""
    dbg = _lib.load_count()
    extra = declared_functions(DEBUG_HEADER)
    assert extra == ["ra_debug_bounds", "ra_debug_ex2_rate", "ra_debug_set_counts"]
    for n in declared_functions() + extra:
        assert hasattr(dbg, n), n
    assert not hasattr(_lib.load(), "ra_debug_set_counts")
    assert not hasattr(_lib.load(), "ra_debug_ex2_rate")
    assert not hasattr(_lib.load(), "ra_debug_bounds")
    assert dbg.ra_debug_bounds(None) == 1
    assert dbg.ra_debug_ex2_rate(0, 1, None, None, None) == 1
    assert dbg.ra_debug_set_counts(None, None) == 0


def test_struct_layout_matches_header():
    assert ctypes.sizeof(_lib.RaTensor) == 8 + 4 + 4 + 32 + 32
    assert ctypes.sizeof(_lib.RaParams) == 4 * 8 + 64 * 4 + 8 + 2 * 8


def test_strerror_covers_codes():
    lib = _lib.load()
    for code in range(0, 12):
        s = lib.ra_strerror(code).decode()
        assert s and s != "unknown error"
    assert lib.ra_strerror(999).decode() == "unknown error"


FAKE = 0x10000  # never dereferenced: validation fails before any device access


def T(shape, dtype=_lib.RA_BF16, strides=None, data=FAKE):
    t = _lib.RaTensor()
    t.data = data
    t.dtype = dtype
    t.ndim = len(shape)
    if strides is None:
        strides, acc = [], 1
        for s in reversed(shape):
            strides.insert(0, acc)
            acc *= s
    for i, (s, st) in enumerate(zip(shape, strides)):
        t.shape[i] = s
        t.stride[i] = st
    return t


def P(qc=128, kc=128, c=1, ring=2, order=None):
    p = _lib.RaParams()
    p.query_chunk_size, p.key_chunk_size, p.causal_block_size, p.ring_size = qc, kc, c, ring
    if order is not None:
        for i, x in enumerate(order):
            p.ring_order[i] = x
        p.use_ring_order = 1
    return p


def fwd(q, k=None, v=None, o=None, lse=None, p=None, bias=None, seg=None, ws=0, ws_bytes=0):
    B, S, H, D = (q.shape[i] for i in range(4))
    k = k or q
    v = v or q
    o = o or T([B, S, H, D], q.dtype)
    lse = lse or T([B, H, S], _lib.RA_F32)
    p = p or P()
    r = lambda x: None if x is None else ctypes.byref(x)
    return _lib.load().ra_forward(ctypes.byref(q), ctypes.byref(k), ctypes.byref(v), r(bias), r(seg),
                                  ctypes.byref(p), ctypes.byref(o), ctypes.byref(lse), ws or None, ws_bytes, None)


def test_forward_argument_errors():
    lib = _lib.load()
    q = T([1, 256, 2, 64])
    assert lib.ra_forward(None, None, None, None, None, None, None, None, None, 0, None) == 1
    assert fwd(T([1, 256, 2, 32])) == 6                                    # head dim 32
    assert fwd(q, k=T([1, 256, 2, 64], _lib.RA_F32)) == 2                   # dtype mismatch
    assert fwd(q, k=T([1, 128, 2, 64])) == 3                                # shape mismatch
    assert fwd(T([1, 256, 2, 64], strides=[256 * 128, 128, 64, 2])) == 4    # head dim not contiguous
    assert fwd(T([1, 256, 2, 64], strides=[256 * 2 * 68, 2 * 68, 68, 1])) == 4   # 136-byte row: TMA rule
    assert fwd(q, p=P(ring=3)) == 5                                         # 256 % 3
    assert fwd(q, p=P(qc=100)) == 5                                         # chunk must divide S/P
    assert fwd(q, p=P(ring=65)) == 6                                        # ring too large
    assert fwd(q, p=P(order=[0, 0])) == 10                                  # not a permutation
    assert fwd(q, p=P(order=[1, 2])) == 10
    seg = T([1, 256], _lib.RA_I32)
    assert fwd(q, seg=seg) == 7                                             # workspace required
    assert fwd(q, seg=T([1, 256], _lib.RA_F32)) == 2                        # segment ids must be int32
    assert fwd(q, bias=T([1, 255], _lib.RA_F32)) == 3
    assert fwd(q, lse=T([1, 2, 256], _lib.RA_BF16)) == 2


def test_empty_inputs_are_a_no_op():
    assert fwd(T([0, 256, 2, 64])) == 0
    assert fwd(T([1, 0, 2, 64]), p=P(qc=1, kc=1)) == 0
    assert fwd(T([1, 256, 0, 64])) == 0


def test_workspace_size_layout():
    lib = _lib.load()
    q = T([2, 1000, 3, 128])
    p = P(qc=500, kc=500, ring=2)
    assert lib.ra_workspace_size(0, ctypes.byref(q), ctypes.byref(p), 0, 0) == 0
    meta = ((2 * 8 * 16 + 255) // 256) * 256      # 8 tiles of 128 tokens per batch row
    assert lib.ra_workspace_size(0, ctypes.byref(q), ctypes.byref(p), 1, 0) == meta
    rows = 2 * 3 * 1024 * 4                        # Delta and lse rows padded to a multiple of 64
    dq = ((2 * 3 * 1000 * 128 * 4 + 255) // 256) * 256
    assert lib.ra_workspace_size(1, ctypes.byref(q), ctypes.byref(p), 0, 1) == meta + 2 * rows + dq
    assert lib.ra_workspace_size(2, ctypes.byref(q), ctypes.byref(p), 0, 0) == ctypes.c_size_t(-1).value


# ---------------------------------------------------------------- host introspection vs oracle

@pytest.mark.parametrize("c", [None, 1, 3, 200])
def test_count_visible_pairs_matches_oracle_integer_mask(c):
    rng = np.random.default_rng(0)
    B, S, H = 2, 700, 3
    seg = np.sort(rng.integers(0, 5, size=(B, S)), axis=1).astype(np.int32)
    seg[1] = rng.integers(0, 3, size=S)           # arbitrary (non-contiguous) ids too
    bias = rng.standard_normal((B, S)).astype(np.float32)
    bias[:, ::7] = -np.inf
    for s_, b_ in ((None, None), (seg, None), (None, bias), (seg, bias)):
        got = api.count_visible_pairs(B, S, H, c, s_, b_)
        want = oracle.visible_pairs_total(B, H, S, c, s_, b_)
        assert got == want


def _visible_tiles(S, rows, c, seg, bias):
    vis = oracle.visible_mask(np.arange(rows[0], rows[1] + 1), S, c, None if seg is None else seg,
                              None if bias is None else bias)
    return {t for t in range((S + 127) // 128) if vis[:, t * 128:(t + 1) * 128].any()}


@pytest.mark.parametrize("S,P,c", [(1024, 4, 1), (1024, 4, None), (2048, 8, 1), (1280, 5, 1), (1000, 2, 7),
                                   (384, 3, None)])
def test_ring_schedule_closes_the_ring(S, P, c):
    """Every visible KV tile is visited exactly once, blocks in ring order (r - t) mod P."""
    blk = S // P
    rng = np.random.default_rng(S + P)
    seg = np.repeat(np.arange(6), S // 6 + 1)[:S].astype(np.int32)
    bias = np.zeros(S, dtype=np.float32)
    bias[rng.integers(0, S, size=S // 3)] = -np.inf
    for sg, bs in ((None, None), (seg, None), (None, bias), (seg, bias)):
        for q_first in range(0, S, 256):
            q_last = min(S - 1, q_first + 255)
            tiles = api.ring_schedule(S, P, q_first, q_last, c, None, sg, bs, blk, blk)
            assert len(tiles) == len(set(tiles)), tiles
            # no visible tile is skipped; skipped ones are invisible to the whole range
            assert _visible_tiles(S, (q_first, q_last), c, sg, bs) <= set(tiles)
            # ring order: blocks appear as r, r-1, r-2, ... (mod P)
            r = q_first // blk
            owner = [(t * 128) // blk for t in tiles]
            steps = [(r - o) % P for o in owner]
            assert steps == sorted(steps), (owner, steps)


def test_ring_schedule_matches_golden_send_receive_table():
    rows = [list(map(int, ln.split())) for ln in open(os.path.join(ROOT, "tests", "golden", "ring_schedule_p4.txt"))
            if ln.strip() and not ln.startswith("#")]
    S, P = 4 * 128, 4                       # one 128-token tile per ring block
    for rank in range(P):
        tiles = api.ring_schedule(S, P, rank * 128, rank * 128 + 127, None)
        assert tiles == [rows[t][1 + rank] for t in range(P)]


def test_ring_schedule_custom_order_is_a_permutation():
    S, P = 1024, 4
    base = api.ring_schedule(S, P, 512, 767, None)
    for order in ([0, 1, 2, 3], [3, 1, 0, 2], [2, 3, 1, 0]):
        tiles = api.ring_schedule(S, P, 512, 767, None, order)
        assert sorted(tiles) == sorted(base)
    with pytest.raises(ValueError):
        api.ring_schedule(S, P, 512, 767, None, [0, 1, 1, 2])


def test_selftest_timeout_rejects_bad_budgets_on_host():
    lib = _lib.load()
    assert lib.ra_selftest_timeout(10, None) == 6          # below the allowed range
    assert lib.ra_selftest_timeout(10 ** 10, None) == 6    # above it


def _host_step(B=1, S=256, H=4, D=64, dtype=_lib.RA_BF16):
    t = _lib.RaHostStep()
    for name in ("q", "k", "v", "d_o", "o", "dq", "dk", "dv", "dev_q", "dev_k", "dev_v", "dev_do", "dev_o", "dev_dq",
                 "dev_dk", "dev_dv"):
        setattr(t, name, T([B, S, H, D], dtype))
    t.lse = T([B, H, S], _lib.RA_F32)
    t.dev_lse = T([B, H, S], _lib.RA_F32)
    return t


def test_train_step_host_argument_errors():
    """ra_train_step_host rejects bad arguments before any stream, event or copy."""
    lib = _lib.load()
    p = P()

    def call(t, hpg=2):
        return lib.ra_train_step_host(ctypes.byref(t) if t is not None else None, None, None, ctypes.byref(p), hpg,
                                      None, 0, None, None, None)

    assert call(None) == 1                                                  # RA_ERR_NULL
    t = _host_step()
    t.dev_dk.data = 0
    assert call(t) == 1                                                     # a missing buffer
    t = _host_step(S=0)
    for name in ("q", "dev_q", "lse"):
        getattr(t, name).data = 0
    assert call(t) == 0                                                     # empty problem: nothing to do
    t = _host_step()
    t.dq = T([1, 256, 4, 64], _lib.RA_F32)
    assert call(t) == 2                                                     # gradients take q's dtype
    t = _host_step()
    t.dev_v = T([1, 128, 4, 64])
    assert call(t) == 3                                                     # device twin of another shape
    t = _host_step()
    t.k = T([1, 256, 4, 64], strides=[256 * 4 * 64, 4 * 64, 64 * 2, 1])   # heads not packed
    assert call(t) == 4                                                     # RA_ERR_STRIDE: not contiguous
    t = _host_step()
    t.lse = T([1, 256, 4], _lib.RA_F32)
    assert call(t) == 3                                                     # lse is [B, H, S]
    t = _host_step()
    assert call(t, hpg=3) == 5                                              # 3 does not divide H = 4
    assert call(t, hpg=0) == 5


def test_plain_c_client(tmp_path):
    """The headers compile as C99 and the host-only entry points work from a C program."""
    import shutil
    import subprocess

    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    pkg = os.path.dirname(_lib.LIB_PATH)
    exe = str(tmp_path / "abi_host_only")
    src = os.path.join(ROOT, "tests", "c", "abi_host_only.c")
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), src, "-o", exe,
                        "-L", pkg, "-lringattn", "-Wl,-rpath," + pkg], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip() == "ok", (r.returncode, r.stdout, r.stderr)


def test_index_check_sites_match_their_documentation():
    """The debug build records out-of-range indices by site number
    (ra_debug_bounds); the header's numbered list of sites must describe the
    RaSite enumeration of the kernels one to one."""
    import os

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    src = open(os.path.join(root, "long_context_exact_ordered_b200", "csrc", "ra_common.cuh")).read()
    body = src[src.index("enum RaSite : int {"):]
    body = body[:body.index("};")]
    names = re.findall(r"\b(kSite\w+)", body)
    assert names[0] == "kSiteFwdTileMeta" and "= 1," in body.split("\n")[1]
    assert len(names) == len(set(names))
    header = open(DEBUG_HEADER).read()
    listing = header[header.index("Sites:"):header.index("int ra_debug_bounds")]
    numbers = sorted(int(n) for n in re.findall(r"(?:^|\s)(\d+) (?:forward|backward|ring step|ring-step|tile|dQ|finalize|feed-forward)",
                                                 listing))
    assert numbers == list(range(1, len(names) + 1)), (numbers, len(names))
    for name in names:   # every site is used by some kernel
        uses = sum(open(os.path.join(root, "long_context_exact_ordered_b200", "csrc", f)).read().count(name)
                   for f in ("ra_common.cuh", "ra_fwd_sm100.cuh", "ra_bwd_sm100.cuh", "ra_simt.cuh", "ra_ffn_sm100.cuh"))
        assert uses >= 2, name
