import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size parity cases (minutes)")


def pytest_collection_modifyitems(config, items):
    # GPU tests without a GPU are skipped only when explicitly deselected;
    # a run that selects them on a machine without CUDA fails loudly.
    pass
