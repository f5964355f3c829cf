"""Plain, slow, fp64 CPU oracle for block-sparse exact softmax attention.

TEST INFRASTRUCTURE ONLY.  Nothing in the library imports this package; only the
tests, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may call it.  It shares no code with the CUDA path.

Contents
--------
``attention``  dense masked softmax attention, its analytic gradient, the fixed-m
               form and the fixed-m bound / per-head gate (plain and k-smoothed).
``bound``      the fixed-m bound per q-block (the reading taken for the pages'
               per-segment kmax): key norms over the kv blocks a q-block reaches.
``blockmap``   the tile classification (EMPTY / PARTIAL / FULL) of a dense mask,
               the kv-column orders, ``rank(m, n)``, the rank-sorted column lists
               and a discrete simulation of the dQ semaphore protocol.

Every function states the passage of the source pages it follows.  Parity pins
live in ``tests/test_oracle_*.py``; no function here is "parity unpinned".
"""

from .attention import (  # noqa: F401
    MaskDesc,
    kv_head_of,
    allowed_rows,
    valid_keys,
    attention_forward,
    attention_backward,
    attention_forward_fixed_m,
    fixed_m_bound,
    fixed_m_bound_smoothed,
    useful_flops,
)
from .bound import fixed_m_bound_blocks, gate_rows_blocks, row_references_blocks  # noqa: F401
from .blockmap import (  # noqa: F401
    EMPTY,
    PARTIAL,
    FULL,
    tile_classes,
    column_order,
    greedy_order,
    kv_ranks,
    column_lists,
    partial_then_full_lists,
    simulate_dq_semaphores,
)
