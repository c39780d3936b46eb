import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(ROOT, "tests", "golden")


def pytest_terminal_summary(terminalreporter):
    """Pooled boundary-excluded code counts of the parity tests that ran (see parity.pooled_check);
    with KVQ_PARITY_RECORD=<path> they are also written there as JSON."""
    try:
        from tests import parity
    except Exception:
        return
    if not parity.POOL:
        return
    rec = {name: parity.pooled(name) for name in sorted(parity.POOL)}
    terminalreporter.write_sep("-", "boundary-excluded codes, pooled per workload (bar: rate < 1e-4)")
    for name, r in rec.items():
        terminalreporter.write_line(f"{name:>18}: {r['excluded']} of {r['coords']} coordinates, rate {r['rate']:.2e}")
    path = os.environ.get("KVQ_PARITY_RECORD")
    if path:
        import json

        with open(path, "w") as f:
            json.dump({"bar": 1e-4, "band": parity.CODE_BAND, "workloads": rec}, f, indent=1)
