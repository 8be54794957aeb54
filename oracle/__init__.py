"""CPU oracle for the streaming int4 MoE block.  TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference arm of
``bench.py`` may import this package.  The product path (the ``libe0moe.so`` library
and its Python binding) never imports, links or runs anything here, and this package
imports nothing from the product path.

Parity pins: every function here is pinned by ``tests/test_oracle_pins.py`` against
closed forms, library routines, invariants or the hand-derived worked example.  No
function is "parity unpinned".
"""
from .moe import *  # noqa: F401,F403
