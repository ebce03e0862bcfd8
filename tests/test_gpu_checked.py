"""The checked build (libdsa_checked.so: the kernels compiled with
-DDSA_DEBUG, whose device-side bounds checks on gathered rows, TMA
coordinates, score writes, cache rows and top-k outputs record error kind 3
and skip the access) runs the workloads of tests/checked_workloads.py with
no error recorded and bit-identical outputs to the release build."""
import json
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_checked_build_records_nothing_and_matches_release():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    lib = os.path.join(ROOT, "sparse_attention_long_07_b200", "libdsa_checked.so")
    if not os.path.exists(lib):
        pytest.fail("libdsa_checked.so is missing: build it with build.py --checked")
    from tests import checked_workloads
    release = checked_workloads.run()
    env = dict(os.environ, DSA_LIBRARY_VARIANT="checked", PYTHONPATH=ROOT)
    out = subprocess.run([sys.executable, "-m", "tests.checked_workloads"], cwd=ROOT, env=env,
                         capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    child = json.loads(out.stdout.strip().splitlines()[-1])
    assert child["library"].endswith("libdsa_checked.so")
    for name, (err, digest) in child["results"].items():
        assert err == 0, f"{name}: checked build recorded {err:#x}"
        assert release[name][0] == 0
        assert digest == release[name][1], f"{name}: outputs differ between builds"
