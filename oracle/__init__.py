"""Test infrastructure: the fp64 CPU oracle for the HLA hot path.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline / reference legs may import
this package.  The product library never does.
"""
from .hla_oracle import *  # noqa: F401,F403
