"""CPU oracle for the SPTS prefill hot path -- TEST INFRASTRUCTURE ONLY.

This package is a plain, slow, fp64 restatement of what the Self-Predictive
Token Skipping (SPTS) prefill layer computes, written from the method's
description in "Probe and Skip: Self-Predictive Token Skipping for Efficient
Long-Context LLM Inference" (Wu et al., 2026): Partial Attention Probing
(Fig. 2(a)), Low-rank Transformation Probing (Fig. 2(b), Table 6, Table A),
the fusion strategies of Table D, and Multi-Stage Delayed Pruning (Fig. 2(c),
Fig. A, Table B).

Who may use it: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py``.  The product
(the CUDA library and its Python binding) never imports, calls or links it,
and it imports nothing from the product: the two share no code.

Every function here has at least one pin in ``tests/test_oracle_pins.py``
(library routines, closed forms, invariants, brute force, or values printed
on the pages).  Functions with no such pin are marked "parity unpinned".
"""

from .spts import *  # noqa: F401,F403
from .accounting import *  # noqa: F401,F403
