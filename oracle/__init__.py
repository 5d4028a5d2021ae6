"""CPU float64 oracle for split-KV decode attention and chunked-prefill attention.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its
CPU-baseline leg and ``--impl reference`` arm) import this package. The CUDA library and its
Python binding never do, and this package imports nothing from them.

* ``attention``    — the plain definition: softmax(q·Kᵀ·scale)·V and its log-sum-exp, decode
                     and chunked-prefill (causal) forms.
* ``formulations`` — the pages' sequential online-softmax and split-then-merge algorithms,
                     used only to pin ``attention``.
* ``planner``      — the split planner the CUDA library must reproduce integer for integer.

Parity status: ``attention`` is pinned by closed forms, hand cases, library routines and
invariants (tests/test_oracle_pins.py); ``planner`` is pinned by coverage / bound properties
and hand-worked plans (tests/test_planner_oracle.py).
"""

from .attention import widen, decode_attention, chunk_prefill_attention, attention_rows  # noqa: F401
from . import formulations, planner  # noqa: F401
