"""Plain fp64 CPU oracle for ring attention (test infrastructure, not product code).

This package exists only to check the CUDA path. Only ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference`` legs
of ``bench.py`` may import it. The product path (``sequence_softmax_b200``) never
imports, links or calls anything here, and nothing here imports the product.

Sources (cited by page title and section):

* "Ring Attention 논문 분석" (youngju.dev blog), listings ``blockwise_attention``,
  ``ring_attention_forward`` and ``ring_attention_causal_step``: the online-softmax
  update and the skip / diagonal / full treatment of a causal KV chunk.
* "Ring Attention" glossary (ultralytics.com, Korean and Vietnamese copies),
  section "How Ring Attention works": the ring visiting order and the 4-device toy
  simulation that must match full softmax attention within 1e-5.
* gpumode lecture 013 notes (brianyu43.github.io), log-sum-exp passage: the
  associativity lse(x) = lse([lse(x1), lse(x2)]); and the causal-imbalance passage
  (striped token placement).
* "Context Parallelism" card (llm-engineer.pages.dev), sections on Ring Attention
  (running max m, running sum l, running output o) and on causal imbalance
  (zig-zag placement).

Backward (gradients of the same attention): ``oracle/backward.py``.

Parity status of every function is stated in its module docstring.
"""

from .backward import attention_backward, backward_rows, delta, partial_backward, ring_backward  # noqa: F401
from .ring import (  # noqa: F401
    NEG_INF,
    attention,
    chunk_class,
    layout_positions,
    merge,
    partial,
    ring_forward,
    toy_ring_unstabilised,
)
