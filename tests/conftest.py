import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def pytest_collection_modifyitems(config, items):
    # Deterministic order: files are collected alphabetically already; keep it.
    return None


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(ROOT, "tests", "golden")


def pytest_terminal_summary(terminalreporter):
    # worst O error over every GPU-vs-oracle comparison of the session (flat bound 2e-2)
    pu = sys.modules.get("parity_utils")
    seen = getattr(pu, "O_OBSERVED", None) if pu else None
    if seen:
        mx = max(x[0] for x in seen)
        mean = max(x[1] for x in seen)
        terminalreporter.write_line(
            f"O parity: {len(seen)} comparisons, worst max-abs {mx:.4e} (bound 2e-2), "
            f"worst mean-abs {mean:.4e} (bound 2e-3)")
