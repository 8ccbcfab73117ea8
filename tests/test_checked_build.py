"""The checked build (libep_a2a_checked.so: device index checks compiled in)
runs in a child process, since a process loads one build of the library."""
import os
import subprocess
import sys

import pytest
import torch

HERE = os.path.dirname(os.path.abspath(__file__))

pytestmark = pytest.mark.gpu


def test_checked_build_matches_the_oracle_and_reports_bad_plan_entries():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from combine_route_plan_b200 import build
    lib = build.build(checked=True)
    env = dict(os.environ, EP_A2A_LIBRARY=lib)
    r = subprocess.run([sys.executable, os.path.join(HERE, "checked_run.py")], env=env,
                       capture_output=True, text=True, timeout=1200)
    assert r.returncode == 0, (r.stdout[-3000:], r.stderr[-3000:])
    assert "checked build ok" in r.stdout
