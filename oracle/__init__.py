"""fp64 CPU oracle of the MoE-layer forward pass (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
and reference legs may import this package; the product path never does.
"""
from .moe_oracle import *  # noqa: F401,F403
from .moe_oracle import HEAVY, IDENTITY, ZERO, CONST  # noqa: F401
