"""Plain fp64 CPU oracle for the WAITS prefill KV-eviction path.

TEST INFRASTRUCTURE ONLY. Nothing in the product package imports this module;
only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its CPU-baseline
and reference legs) may import or call it. It shares no code, tables or
helpers with the CUDA library: both sides receive the same arrays from the
seeded input generators and nothing else.

Every function restates its source on the WAITS README page
(stig.sh/Dirac-Notation/A2SF): the opening summary defines the forgetting
curve and the accumulative score, the Quickstart defines ``recent_budget`` and
``select_budget``.

Pinned by ``tests/test_oracle_pins.py`` (decimal brute force, closed forms,
limits, invariants) and ``tests/test_oracle_select_compact.py`` (textbook
sort, explicit loops). No function here is "parity unpinned".
"""

from .waits_oracle import (  # noqa: F401
    forgetting_curve,
    row_lse,
    score,
    select,
    compact,
    compress,
    decode_attention,
)
