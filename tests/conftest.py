import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 and the built CUDA library")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def pytest_terminal_summary(terminalreporter):
    # near-tie counts and worst errors the parity tests recorded (tests/parity_util.py REPORT)
    mod = sys.modules.get("parity_util")
    lines = getattr(mod, "REPORT", None) if mod else None
    if lines:
        terminalreporter.write_sep("-", "parity report")
        for line in lines:
            terminalreporter.write_line(line)
