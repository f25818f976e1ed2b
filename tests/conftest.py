import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def read_golden(name):
    """Lines of a golden fixture with comments and blank lines removed."""
    out = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                out.append(line)
    return out


@pytest.fixture(scope="session")
def golden():
    return read_golden


def pytest_terminal_summary(terminalreporter):
    """Per test: the parity margins the GPU checks observed (largest
    estimate error / tolerance, tolerated Top-k disagreements, largest
    attention error / tolerance)."""
    parity = sys.modules.get("tests.parity")
    if parity is None or not parity.STATS:
        return
    tr = terminalreporter
    tr.section("parity margins (error / tolerance; Top-k disagreements)")
    tr.write_line("%-72s %6s %6s %9s %9s" % ("test", "pairs", "swaps", "est", "attn"))
    for test, s in sorted(parity.STATS.items()):
        tr.write_line("%-72s %6d %6d %9.2e %9.2e" % (test[-72:], s["pairs"], s["swaps"], s["est"], s["attn"]))
