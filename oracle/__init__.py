"""CPU oracle for the NVFP4 W4A4 path -- test infrastructure only.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline and
reference legs import this package. The CUDA library never does.
"""
from .nvfp4_oracle import *  # noqa: F401,F403
