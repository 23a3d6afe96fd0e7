"""CPU oracle for the NVFP4 routed-expert MoE chain.

TEST INFRASTRUCTURE ONLY: the tests, the package smoke check and the CPU
baseline leg of bench.py may import this package; the product path never does.
The arithmetic lives in oracle.c; this module only marshals numpy arrays.
"""
from .oracle import *  # noqa: F401,F403
