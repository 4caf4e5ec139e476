import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

# Mask-parity records of the GPU tests, printed at the end of the run: per
# case, the rows compared, the rows the oracle flags as near ties, the rows
# whose kept set differs from the oracle's (allowed only in near-tie rows)
# and, where the test ran it, the end-to-end comparison (the oracle pooling
# and scoring by itself).
_MASK_PARITY = []


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size configuration")


@pytest.fixture(scope="session")
def orc():
    from oracle import oracle
    oracle.build_oracle()
    return oracle


@pytest.fixture(scope="session")
def mask_report():
    """List of dicts, one per mask comparison; see pytest_terminal_summary."""
    return _MASK_PARITY


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    if not _MASK_PARITY:
        return
    tr = terminalreporter
    tr.section("mask parity: GPU kv lists against the oracle's selection")
    small = [r for r in _MASK_PARITY if not r.get("full_size")]
    if small:
        tr.write_line("small cases: {} comparisons, {} rows, {} near-tie rows, {} differing rows, "
                      "{} differing outside the near-tie band".format(
                          len(small), sum(r["rows"] for r in small), sum(r["near_tie_rows"] for r in small),
                          sum(r["mismatched_rows"] for r in small), sum(r["unexcused"] for r in small)))
    for r in _MASK_PARITY:
        if not r.get("full_size"):
            continue
        line = ("{case}: {rows} rows, {near_tie_rows} near-tie, {mismatched_rows} differing, "
                "{unexcused} outside the band".format(**r))
        if "e2e_rows" in r:
            line += ("; end to end (oracle pools and scores itself) on {e2e_heads} heads: {e2e_rows} rows, "
                     "{e2e_mismatched_rows} differing".format(**r))
        tr.write_line(line)
