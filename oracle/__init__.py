"""CPU float64 oracle of the CalibAtt hot path: test infrastructure only.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline legs import
this package; the product package never does.
"""
from .calibatt_oracle import *  # noqa: F401,F403
