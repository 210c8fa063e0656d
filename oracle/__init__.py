"""CPU oracle for the AWQ per-layer scale search — TEST INFRASTRUCTURE ONLY.

This package is the plain, slow, obviously correct statement of what the search
computes. It shares no code with the CUDA path and neither imports the other. Only
``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline / reference
arm may import it; the product path (``post_quantization_column_b200``) never does
and fails loudly when its CUDA library is missing.

Parity pins: every function here is checked in ``tests/test_oracle_pins.py`` against
values the pages print (the two-channel worked example), closed forms, invariants
and brute force. See ``awq_oracle``'s docstring for which pin covers which step.
"""
from .awq_oracle import *  # noqa: F401,F403
