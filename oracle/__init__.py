"""fp64 CPU oracle of the routed-MoE FFN step (test infrastructure only).

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may import
this package. The product library never does. Parity of every function here
is pinned by the tests in tests/test_oracle_pins.py (hand-computed dequant bit
patterns, closed-form routing and SwiGLU values, brute force over all top-k
subsets, dense masked evaluation of every expert); the end-to-end layer output
has no value printed on the pages to pin it against, so beyond those pins its
parity with the pages is unpinned.
"""
from .moe_oracle import *  # noqa: F401,F403
