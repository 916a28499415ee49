"""Seeded synthetic workloads shared by the oracle side and the CUDA side.

This package only draws numbers and lays them out in the byte formats the
caches use. It holds none of the method's arithmetic: no pooling, no norm, no
rotation, no scoring, no attention.
"""

from .workloads import *  # noqa: F401,F403
