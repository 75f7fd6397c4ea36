"""The bounds-checking debug build (liblmoe_checks.so, built with
-DLMOE_CHECKS): small parity cases and the checks themselves, run in a child
process that loads the debug build through LMOE_LIBRARY (tests/checks_cases.py)."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_debug_build_parity_and_bounds_checks():
    import importlib.util
    spec = importlib.util.spec_from_file_location("lmoe_build", os.path.join(ROOT, "latentmoe_fwd_b200", "build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    lib = b.build(checks=True)
    env = dict(os.environ, LMOE_LIBRARY=lib)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "checks_cases.py")], env=env,
                       capture_output=True, text=True, timeout=900, cwd=ROOT)
    print(r.stdout[-4000:])
    print(r.stderr[-4000:])
    assert r.returncode == 0 and "CHECKS_OK" in r.stdout
