import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200) and the built library")
    config.addinivalue_line("markers", "slow: large CPU oracle runs")
    config.addinivalue_line("markers", "integration: checks composed from the parity cases (shardings, buffer "
                                       "guards); collected after the plain parity tests")
    config.addinivalue_line("markers", "fullsize: benchmark-sized workloads; collected after every other test")


def pytest_collection_modifyitems(session, config, items):
    # Plain parity cases first, then the checks built on them, then the benchmark-sized
    # cases (the longest, and the largest allocations): a run stopped at the first failure
    # has still reported everything before it.
    # The no-workspace entry point's test file (test_zz_*) goes after everything else.
    def rank(it):
        if os.path.basename(str(it.fspath)).startswith("test_zz_"):
            return 3
        if it.get_closest_marker("fullsize") is not None:
            return 2
        return 1 if it.get_closest_marker("integration") is not None else 0
    items.sort(key=rank)
