import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Near-tie allowances the GPU/oracle comparisons used in this run."""
    mod = sys.modules.get("tests.parity")
    if mod is None or not mod.TOTALS["segments"]:
        return
    t = mod.TOTALS
    terminalreporter.write_line(
        f"near-tie allowances: {t['swapped_positions']} order positions (|ds| <= 1e-6 max|s|) and "
        f"{t['C_flips']} stop blocks (|m - tau| <= 1e-6 tau) over {t['segments']} compared segment plans; "
        f"{t['online_C_flips']} run-time stop flips")
