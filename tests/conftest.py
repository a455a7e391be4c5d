import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
# every binding call in the tests reads back its device status word and raises on a finding
# (tests that provoke one on purpose pass check_status=False)
os.environ.setdefault("GDN_CHECK_STATUS", "1")
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
