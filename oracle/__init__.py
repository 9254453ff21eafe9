"""fp64 CPU oracle of the hybrid attention chunk step (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may import this package. The product path never does.
"""
from .hf_oracle import *  # noqa: F401,F403
from .hf_oracle import __all__  # noqa: F401
