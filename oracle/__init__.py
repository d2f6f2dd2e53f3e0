"""ORACLE — test infrastructure, not product code.

A plain single-threaded fp64 C++ statement of the LSRM native-sparse-attention
layer (nsa_oracle.cpp) and a ctypes wrapper (oracle.py).  Only the tests, the
smoke check and the benchmark's CPU-baseline leg load it.  It shares no code
with the CUDA path; the only module both sides use is the seeded input
generator in ``workloads``.
"""
from .oracle import *  # noqa: F401,F403
