"""CPU oracle of the partitioned Transformer layer (test infrastructure only).

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline and
reference legs may import this package.  The product path never does.
"""
from . import tp_oracle  # noqa: F401
