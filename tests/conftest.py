import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Print the measured parity figures of every GPU comparison that ran."""
    mod = sys.modules.get("parity_util")
    if mod is None:
        return
    tr = terminalreporter
    if mod.REPORT:
        tr.write_sep("-", "forward parity (CUDA vs fp64 oracle)")
        tr.write_line(f"{'case':60s} {'max|dO|':>10s} {'mean|dO|':>10s} {'max rel dLSE':>13s}")
        for what, mx, mean, dl in mod.REPORT:
            tr.write_line(f"{what[:60]:60s} {mx:10.3e} {mean:10.3e} {dl:13.3e}")
    if mod.GRAD_REPORT:
        tr.write_sep("-", "backward parity (CUDA vs fp64 oracle, per-slice rms units)")
        tr.write_line(f"{'case':60s} {'max excess':>11s} {'mean':>10s}")
        for what, ex, mean in mod.GRAD_REPORT:
            tr.write_line(f"{what[:60]:60s} {ex:11.3e} {mean:10.3e}")
