"""fp64 CPU oracle for SLAY spherical Yat-kernel linear attention.

TEST INFRASTRUCTURE ONLY.  The tests, the package smoke check and the benchmark's
CPU-baseline leg may import this package; the library's product path never does.
"""
from .oracle import *  # noqa: F401,F403
