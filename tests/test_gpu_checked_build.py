"""The checked build (PKV_CHECK=1, libpariskv_check.so): the same kernels with extra
device-side checks that record ST_BADINDEX and skip the access, never trap. The stage
parity tests and the check tests run against it in a child process (the binding picks the
library when it is imported), so they pass with every check compiled in."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
pytestmark = pytest.mark.gpu


def test_parity_and_check_tests_pass_on_the_checked_build():
    from long_context_kv_srht_b200 import build as kbuild
    lib = kbuild.build(check=True)
    env = dict(os.environ, PARISKV_LIBRARY="check")
    probe = subprocess.run([sys.executable, "-c",
                            "from long_context_kv_srht_b200 import pariskv as pk; "
                            "print(pk.LIB_PATH)"], env=env, cwd=ROOT, capture_output=True,
                           text=True, timeout=300)
    assert probe.returncode == 0 and probe.stdout.strip() == lib, probe.stderr[-2000:]
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        "tests/test_gpu_parity.py", "tests/test_gpu_checks.py", "-k",
                        "stages_bit_exact or adversarial or tiny_query or sparse_attend or "
                        "group_union or bad_candidate or launch_shape"],
                       env=env, cwd=ROOT, capture_output=True, text=True, timeout=1500)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    assert " passed" in r.stdout and " failed" not in r.stdout
