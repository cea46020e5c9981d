import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
for _p in (ROOT, os.path.join(ROOT, "tests")):
    if _p not in sys.path:
        sys.path.insert(0, _p)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    # The in-tree CUDA library must match the sources before the package is imported: a
    # fresh checkout has no libfocus.so (the oracle builds itself on first use).  Nothing
    # happens when it is up to date.
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_focus_build", os.path.join(ROOT, "attention_delta_token_b200", "build.py"))
    builder = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(builder)
    builder.build()


@pytest.fixture(scope="session")
def orc():
    import oracle
    return oracle.default()


# Per-config selection reports of the parity tests (how many kept sets were
# checked exactly, how many fell in the tie band), printed after the run.
PARITY_REPORT = []


@pytest.fixture(scope="session")
def parity_report():
    return PARITY_REPORT


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    if PARITY_REPORT:
        terminalreporter.section("selection parity (kept sets checked against the oracle)")
        for line in PARITY_REPORT:
            terminalreporter.write_line(line)
