"""CPU oracle for the event-tensor hot path.

TEST INFRASTRUCTURE ONLY: imported by the tests, by the smoke check and by
the benchmark's CPU-baseline leg, never by the product package.  It shares
no code with the CUDA path.  The arithmetic lives in ``oracle.c`` (plain C,
double accumulation); ``dag.py`` expands event-tensor task graphs by brute
force.
"""
from .api import *  # noqa: F401,F403
from . import dag  # noqa: F401
