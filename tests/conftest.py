import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: takes more than a few seconds on CPU")


@pytest.fixture(scope="session")
def oracle_lib():
    import oracle
    return oracle.load()


@pytest.fixture(scope="session")
def parity_log():
    """Appends one JSON record per call to the file named by TESSERA_PARITY_LOG
    (when set): the whole-tensor error figures of the every-element checks."""
    import json
    path = os.environ.get("TESSERA_PARITY_LOG")

    def record(**fields):
        if path:
            with open(path, "a") as f:
                f.write(json.dumps(fields) + "\n")
    return record
