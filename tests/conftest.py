import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

# (test, quantity, worst rel-L2 / rel-Fro, worst max-abs, worst head, tolerance)
# rows appended by the parity tests, printed at the end of the session
MARGINS = []


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 GPU and the built CUDA library")


def pytest_terminal_summary(terminalreporter):
    if not MARGINS:
        return
    terminalreporter.write_sep("-", "parity margins (worst over heads)")
    for name, what, rel, mx, head, tol in MARGINS:
        terminalreporter.write_line(
            f"{name:<34} {what:<22} rel {rel:.3e}  max-abs {mx:.3e}  head {head:>3}  tol {tol}")
