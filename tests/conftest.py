import os
import sys
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parent.parent
if str(ROOT) not in sys.path:
    sys.path.insert(0, str(ROOT))


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: longer-running CPU test")


@pytest.fixture(autouse=True)
def _parity_test_name(request):
    # the O checks record which test they ran in (tests/tolerance.py)
    from tests import tolerance

    tolerance.CURRENT_TEST = request.node.nodeid
    yield


def pytest_terminal_summary(terminalreporter):
    from tests import tolerance

    lines = tolerance.o_summary()
    if lines:
        terminalreporter.write_sep("-", "O parity: storage floor and elements passed on the bf16 allowance")
        for line in lines:
            terminalreporter.write_line(line)
