"""CPU float64 oracle of Maglev's injected sliding-window attention.

TEST INFRASTRUCTURE ONLY: imported by tests/, __graft_entry__.smoke() and the
CPU-baseline legs of bench.py, never by the CUDA path.
"""
from .maglev_oracle import *  # noqa: F401,F403
