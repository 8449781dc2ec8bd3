"""CPU oracle of the DSA sparse-attention path -- test infrastructure only.

Imported by the tests, by ``__graft_entry__.smoke()`` and by the CPU-baseline
leg of ``bench.py``; never by the product path.
"""
from .dsa_oracle import *  # noqa: F401,F403
from . import dsa_oracle  # noqa: F401
