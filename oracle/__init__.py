"""CPU oracle of the ARL2 hybrid-attention hot path (test infrastructure only).

Imported by the tests, by ``__graft_entry__.smoke()`` and by the benchmark's
CPU-baseline leg; never by the CUDA path.
"""
from . import arl2_oracle, brute  # noqa: F401
