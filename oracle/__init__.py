"""Plain CPU oracle for rank-major MoE EP dispatch / combine.

TEST INFRASTRUCTURE ONLY: imported by the test suite, by the smoke check in
``__graft_entry__`` and by the benchmark's CPU-baseline leg, never by the
product path.  It shares no code with the CUDA library.
"""
from .oracle import *  # noqa: F401,F403
