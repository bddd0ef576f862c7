"""CPU oracle of the HGRNBit block forward. TEST INFRASTRUCTURE: imported only by tests/,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``; never by the product path."""
from .mmf_oracle import *  # noqa: F401,F403
