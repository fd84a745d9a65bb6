"""ctypes declarations for ``libringattn.so`` (the C ABI in include/ringattn.h).

Loading fails loudly: there is no Python or CPU fallback for any entry point.
"""

from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libringattn.so")
# Debug build (-DRA_DEBUG_COUNT): same entry points plus ra_debug_set_counts.
COUNT_LIB_PATH = os.path.join(HERE, "libringattn_count.so")

RA_F32, RA_BF16, RA_I32 = 0, 1, 2
RA_MAX_RING = 64

ERRORS = {
    0: "RA_OK", 1: "RA_ERR_NULL", 2: "RA_ERR_DTYPE", 3: "RA_ERR_SHAPE", 4: "RA_ERR_STRIDE",
    5: "RA_ERR_DIVISIBILITY", 6: "RA_ERR_UNSUPPORTED", 7: "RA_ERR_WORKSPACE", 8: "RA_ERR_CUDA",
    9: "RA_ERR_DEVICE_TIMEOUT", 10: "RA_ERR_ORDER", 11: "RA_ERR_STATIC_LIMIT",
}


class RaTensor(ctypes.Structure):
    _fields_ = [
        ("data", ctypes.c_void_p),
        ("dtype", ctypes.c_int32),
        ("ndim", ctypes.c_int32),
        ("shape", ctypes.c_int64 * 4),
        ("stride", ctypes.c_int64 * 4),
    ]


class RaParams(ctypes.Structure):
    _fields_ = [
        ("query_chunk_size", ctypes.c_int64),
        ("key_chunk_size", ctypes.c_int64),
        ("causal_block_size", ctypes.c_int64),
        ("ring_size", ctypes.c_int64),
        ("ring_order", ctypes.c_int32 * RA_MAX_RING),
        ("use_ring_order", ctypes.c_int32),
        ("reserved", ctypes.c_int32),
        ("prof_event_begin", ctypes.c_void_p),
        ("prof_event_end", ctypes.c_void_p),
    ]


class RaHostStep(ctypes.Structure):
    _fields_ = [(n, RaTensor) for n in ("q", "k", "v", "d_o", "o", "lse", "dq", "dk", "dv", "dev_q", "dev_k", "dev_v",
                                         "dev_do", "dev_o", "dev_lse", "dev_dq", "dev_dk", "dev_dv")]


_T = ctypes.POINTER(RaTensor)
_P = ctypes.POINTER(RaParams)
_vp = ctypes.c_void_p

SIGNATURES = {
    "ra_workspace_size": (ctypes.c_size_t, [ctypes.c_int, _T, _P, ctypes.c_int, ctypes.c_int]),
    "ra_forward": (ctypes.c_int, [_T, _T, _T, _T, _T, _P, _T, _T, _vp, ctypes.c_size_t, _vp]),
    "ra_forward_static": (ctypes.c_int, [_T, _T, _T, _T, _T, _P, _T, _T, _vp]),
    "ra_backward": (ctypes.c_int, [_T, _T, _T, _T, _T, _T, _T, _T, _P, _T, _T, _T, _vp, ctypes.c_size_t, _vp]),
    "ra_step": (ctypes.c_int, [_T, _T, _T, ctypes.c_int64, ctypes.c_int64, _T, _T, _T, _P, _T, _T, _T, _vp]),
    "ra_finalize": (ctypes.c_int, [_T, _T, _T, _T, _T, _vp]),
    "ra_lse_merge": (ctypes.c_int, [_T, _T, _T, _T, _T, _T, _vp]),
    "ra_train_step_host": (ctypes.c_int, [ctypes.POINTER(RaHostStep), _T, _T, _P, ctypes.c_int64, _vp,
                                          ctypes.c_size_t, _vp, _vp, _vp]),
    "ra_feedforward_workspace_size": (ctypes.c_size_t, [ctypes.c_int64, ctypes.c_int64]),
    "ra_feedforward": (ctypes.c_int, [_T, _T, _T, _T, _T, ctypes.c_int64, _vp, ctypes.c_size_t, _vp]),
    "ra_get_device_status": (ctypes.c_int, [_vp]),
    "ra_selftest_timeout": (ctypes.c_int, [ctypes.c_int64, _vp]),
    "ra_strerror": (ctypes.c_char_p, [ctypes.c_int]),
    "ra_last_error_message": (ctypes.c_char_p, []),
    "ra_count_visible_pairs": (ctypes.c_int64, [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                                 ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_float)]),
    "ra_ring_schedule": (ctypes.c_int64, [ctypes.c_int64, _P, ctypes.c_int64, ctypes.c_int64,
                                           ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_float),
                                           ctypes.POINTER(ctypes.c_int32), ctypes.c_int64]),
}

_lib = None


def load() -> ctypes.CDLL:
    """Load the shared library once; raise if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with `python -m long_context_exact_ordered_b200.build` "
                "(there is no fallback implementation)")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


_count_lib = None


def load_count() -> ctypes.CDLL:
    """Load the debug build (kernels that also count visible pairs); raise if absent."""
    global _count_lib
    if _count_lib is None:
        if not os.path.exists(COUNT_LIB_PATH):
            raise ImportError(f"{COUNT_LIB_PATH} is missing: build it with `python -m long_context_exact_ordered_b200.build`")
        lib = ctypes.CDLL(COUNT_LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        lib.ra_debug_set_counts.restype = ctypes.c_int
        lib.ra_debug_set_counts.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
        lib.ra_debug_ex2_rate.restype = ctypes.c_int
        lib.ra_debug_ex2_rate.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p,
                                          ctypes.c_void_p]
        lib.ra_debug_bounds.restype = ctypes.c_int
        lib.ra_debug_bounds.argtypes = [ctypes.POINTER(ctypes.c_uint64)]
        _count_lib = lib
    return _count_lib


def swap(lib):
    """Make ``lib`` the library every later call goes to; return the previous one."""
    global _lib
    prev = load()
    _lib = lib
    return prev


class RingAttnError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        msg = load().ra_strerror(code).decode()
        if code == 8:                                  # RA_ERR_CUDA: which call failed, and how
            detail = load().ra_last_error_message().decode()
            if detail:
                msg = f"{msg}: {detail}"
        super().__init__(f"{where}: {ERRORS.get(code, code)} ({msg})")


def check(code: int, where: str):
    if code != 0:
        raise RingAttnError(code, where)
