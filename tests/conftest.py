import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200) and the built library")
    config.addinivalue_line("markers", "slow: large CPU oracle runs")
    config.addinivalue_line("markers", "fullsize: benchmark-sized workloads; collected after every other test")


def pytest_collection_modifyitems(session, config, items):
    # The benchmark-sized cases take the longest and allocate the most; run them after
    # the small parity cases so that a run stopped at the first failure still reports those.
    items.sort(key=lambda it: it.get_closest_marker("fullsize") is not None)
