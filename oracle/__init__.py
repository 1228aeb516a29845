"""fp64 CPU oracle of the RRAttention prefill hot path (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline / reference arm
may import this package. The product path never does.
"""
from .rr_oracle import *  # noqa: F401,F403
from .rr_oracle import __all__  # noqa: F401
