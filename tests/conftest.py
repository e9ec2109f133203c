import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
HERE = os.path.dirname(os.path.abspath(__file__))
if HERE not in sys.path:
    sys.path.insert(0, HERE)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    # achieved errors of every GPU-vs-oracle comparison of this run (tests/parity_check.py)
    mod = sys.modules.get("parity_check")
    if mod is None or not mod.MARGINS:
        return
    terminalreporter.write_sep("-", "parity margins (GPU against the fp64 oracle)")
    for line in mod.MARGINS:
        terminalreporter.write_line(line)
