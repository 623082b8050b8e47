"""Float64 CPU oracle of the VDN-H3 linear branch (test infrastructure only).

Only tests/, the package smoke check and the benchmark's CPU-baseline leg use it.
"""
from .vdn_oracle import *  # noqa: F401,F403
