"""CPU oracle for Ring Attention's blockwise exact attention.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute anything in this package; only the tests, ``__graft_entry__.smoke()``
and the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.
It shares no code with the CUDA path: it does not import the product package
and the product package does not import it.

Sources (the pages describing the method, cited by title and section):

* [RA-tech]  "Ring Attention技术解析：突破大模型长上下文训练瓶颈",
  §2.1 (the N×N attention matrix), §2.2 (ring of devices, send to the next
  rank / receive from the previous one).
* [RA-LWM]   "手把手拆解RingAttention：如何用分布式计算突破百万token长视频处理瓶颈",
  §1 (the complexity table: RingAttention keeps global attention complete;
  queries stay, key/value blocks travel round the ring).
* [RA-core]  "RingAttention核心功能全解析", headings 核心技术原理 1 (query/key
  chunk sizes, ``causal_block_size``), 核心API调用 (``ringattention(xq, xk,
  xv, attention_bias, segment_ids, blockwise_kwargs)`` and the
  ``nothing_saveable`` recompute policy).

Modules
-------
``attention``  the plain definition of masked softmax attention and its
               analytic backward, float64 numpy (the oracle proper).
``loops``      the same definition as pure-Python loops for tiny inputs
               (an independent restatement used to pin ``attention``).
``feedforward`` the blockwise feed-forward network (SwiGLU) exported next
               to ``ringattention``.
``ring``       the ring-blockwise path (P virtual ranks, chunked online
               softmax, log-sum-exp merge): a second, independent route to
               the same numbers, used only by the oracle's self-tests.

Pinned by tests/test_oracle_pins.py (brute force, closed forms, invariances,
finite differences, a library routine, and a negative control).
"""

from .attention import (  # noqa: F401
    attention_backward,
    attention_forward,
    attention_rows,
    backward_term_magnitudes,
    causal_ok,
    head_backward_cols,
    visible_count_cols,
    visible_count_rows,
    visible_mask,
    visible_pairs_total,
)
from .feedforward import blockwise_feedforward, silu  # noqa: F401
from .ring import finalize, lse_merge, online_step, ring_blockwise_reference  # noqa: F401
