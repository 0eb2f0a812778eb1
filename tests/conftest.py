import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    os.environ.setdefault("YR_WAIT_TIMEOUT_MS", "2000")
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU")


@pytest.fixture(scope="session")
def golden():
    import json
    path = os.path.join(ROOT, "tests", "golden")

    def load(name):
        with open(os.path.join(path, name)) as f:
            return json.load(f)
    return load
