"""B200-native Ring Attention: blockwise exact attention over virtual ring ranks.

The compute path is ``libringattn.so`` (hand-written sm_100a CUDA behind a C
ABI, include/ringattn.h); this package only marshals torch tensors into it.
"""

from .api import (  # noqa: F401
    HostStep,
    RingAttentionFunction,
    blockwise_feedforward,
    count_visible_pairs,
    device_status,
    finalize,
    init_state,
    lse_merge,
    ring_schedule,
    ring_step,
    ringattention,
    ringattention_backward,
    ringattention_static,
    selftest_timeout,
    visible_count_probe,
    workspace_size,
)
from ._lib import RingAttnError, load  # noqa: F401

__all__ = [
    "ringattention", "ringattention_backward", "ringattention_static", "ring_step", "init_state", "finalize", "lse_merge",
    "device_status", "selftest_timeout", "count_visible_pairs", "ring_schedule", "workspace_size", "RingAttentionFunction", "visible_count_probe",
    "HostStep", "RingAttnError", "load", "blockwise_feedforward",
]
