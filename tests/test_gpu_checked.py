"""The checked build (-DGDR_CHECK, libgdr_check.so) on the GPU: its bounds
self-test reports GDR_ERR_BOUNDS without touching memory, no guard fires on any
valid call of any entry point, and every output is bit-identical to the normal
library's (the guards only read indices)."""
import os
import subprocess
import sys

import numpy as np
import pytest

from gated_delta_rule_90_b200 import binding

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))


def test_checked_build_matches_normal_build(cuda_device, tmp_path):
    if not os.path.exists(binding.CHECKED_LIB_PATH):
        from gated_delta_rule_90_b200 import build
        build.build(checked=True)
    import checked_cases
    assert not binding.checked_build()
    assert binding.selftest_bounds() == binding.GDR_ERR_UNSUPPORTED
    ref = checked_cases.run_cases(cuda_device)
    path = str(tmp_path / "checked.npz")
    root = os.path.dirname(HERE)
    env = dict(os.environ, GDR_LIBRARY=binding.CHECKED_LIB_PATH,
               PYTHONPATH=os.pathsep.join(p for p in (root, os.environ.get("PYTHONPATH")) if p))
    r = subprocess.run([sys.executable, os.path.join(HERE, "checked_cases.py"), path], env=env,
                       cwd=root, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    got = np.load(path)
    assert sorted(got.files) == sorted(ref)
    for name, x in ref.items():
        assert np.array_equal(got[name], x, equal_nan=True), name
