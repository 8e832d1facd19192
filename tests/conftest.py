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


# Parity reports (selection rows that differ from the oracle only inside the
# tie band; rows the on-chip selection left to the exact kernel) are emitted
# as TieBandReport warnings by tests/parity.py and the GPU parity tests; they
# are gathered here and repeated as one section at the end of the run, just
# above the final counts, so that a short tail of the log shows them.
_PARITY_REPORTS = []


def pytest_warning_recorded(warning_message, when, nodeid, location):
    if warning_message.category.__name__ == "TieBandReport":
        _PARITY_REPORTS.append(str(warning_message.message))


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    if _PARITY_REPORTS:
        terminalreporter.section("parity reports (tie band; rows finished by the exact kernel)")
        for line in _PARITY_REPORTS:
            terminalreporter.write_line(line)
