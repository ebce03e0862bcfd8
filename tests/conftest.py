import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def oracle_lib():
    import oracle
    oracle.build()
    return oracle


def build_library():
    """Compile libdsa.so if stale (the builder is loaded by path, not through the package)."""
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "dsa_build", os.path.join(ROOT, "sparse_attention_long_07_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.build()


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Largest error-to-limit fractions seen by the parity checks of this session."""
    try:
        from tests import parity
    except ImportError:
        return
    if not parity.MARGINS:
        return
    worst = {}
    for what, ratio in parity.MARGINS:
        key = what.split(" (")[0]
        if ratio >= worst.get(key, (-1.0, ""))[0]:
            worst[key] = (ratio, what)
    terminalreporter.write_sep("-", "parity margins (worst error / limit; 1.0 = at the limit)")
    for key, (ratio, what) in sorted(worst.items()):
        terminalreporter.write_line(f"{key:18s} {ratio:.4f}   [{what}]")
