import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
# The mutation tests (tests/test_oracle_mutants.py) run the pins against a
# copy of the oracle package with one planted mistake: VEDA_ORACLE_DIR names
# the folder holding that copy, which then shadows the repository's oracle.
_ALT_ORACLE = os.environ.get("VEDA_ORACLE_DIR")
if _ALT_ORACLE:
    sys.path.insert(0, _ALT_ORACLE)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_report_header(config):
    if _ALT_ORACLE:
        return f"oracle package from VEDA_ORACLE_DIR={_ALT_ORACLE}"
    return None


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    if _ALT_ORACLE:
        assert oracle.__file__.startswith(_ALT_ORACLE), oracle.__file__
    oracle.build()
    return oracle
