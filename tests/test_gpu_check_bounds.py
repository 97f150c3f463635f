"""The HYENA_CHECK_BOUNDS debug build (libhyena_checked.so): the same kernels
with every checked index verified on the device. Small and odd shapes through
each forward family must match the oracle with no check failing; the cases run
in a process of their own, which loads the checked library."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


def test_checked_build_small_and_odd_shapes():
    from long_convolution_sequence_hyena_b200 import build
    lib = build.build(checked=True)
    assert os.path.exists(lib)
    env = dict(os.environ, HYENA_LIBRARY="checked")
    out = subprocess.run([sys.executable, os.path.join(HERE, "check_bounds_cases.py")], env=env,
                         capture_output=True, text=True, timeout=900)
    assert out.returncode == 0 and out.stdout.strip().endswith("OK"), (out.stdout[-2000:], out.stderr[-4000:])
