"""The bounds-checked build (libra_checked.so, RA_DEBUG_BOUNDS): every global row index and
TMA start row the kernels compute is tested against its buffer, and a failure is recorded
in the device error word instead of touching memory. On representative calls of every entry
point (tests/checked_cases.py) no test fires, and the outputs equal the default build's bit
for bit -- the checks only guard, they never change the arithmetic. (The pool's sanitizer is
closed; this is the substitute.)"""

import os
import subprocess
import sys

import numpy as np
import pytest

from sequence_softmax_b200 import build

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_checked_build_matches_default(cuda, tmp_path):
    from . import checked_cases

    lib = build.build(checked=True)
    out = tmp_path / "checked.npz"
    env = dict(os.environ, RA_LIBRARY=lib, PYTHONPATH=ROOT + os.pathsep + os.environ.get("PYTHONPATH", ""))
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "checked_cases.py"), str(out)], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    got = np.load(out)
    ref = checked_cases.run_cases()  # this process has the default library loaded
    for name, arrays in ref.items():
        for i, a in enumerate(arrays):
            b = got[f"{name}|{i}"]
            assert np.array_equal(a, b, equal_nan=True), f"{name}[{i}] differs between checked and default builds"
