"""The bounds-checked debug build (-DSAD_CHECKS, libsad_checks.so) gives the
oracle's results on tiny, ragged, crowded and duplicate-id cases, and its
device-side checks refuse no access there.  It runs in a child process: the
library is chosen when the binding first loads it."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


def test_checked_build_refuses_no_access():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    env = dict(os.environ, SAD_CHECKS="1")
    r = subprocess.run([sys.executable, os.path.join(HERE, "checked_cases.py")], env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    res = json.loads(r.stdout.strip().splitlines()[-1])
    assert res["cases"] == 5 and res["check_failures"] == 0, res
    # two of the cases take the TMA-staged form (2 and 6 tiles); with their
    # first copies withheld every block fell back to plain loads
    assert res["withheld_fallbacks"] == 8, res
    # the full-size workload, generic path included, refuses no access either
    assert res["full_size"] == 0, res
