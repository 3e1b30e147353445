import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Top-k gap certificates and near-tie swap counts of the parity tests."""
    lib = sys.modules.get("hylra_testlib")
    lines = lib.certificate_lines() if lib is not None else []
    if lines:
        terminalreporter.write_sep("-", "top-k gap certificates (oracle fp32 scores)")
        for line in lines:
            terminalreporter.write_line(line)
