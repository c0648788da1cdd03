import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """The achieved parity errors (max |gpu - ref| / max |ref|), the largest per test, so that the
    margin under each bar is visible in every run and not only when a test fails."""
    mod = sys.modules.get("parity_util")
    rows = getattr(mod, "ACHIEVED", None) if mod is not None else None
    if not rows:
        return
    worst = {}
    for test, e in rows:
        worst[test] = max(e, worst.get(test, 0.0))
    terminalreporter.write_sep("-", "achieved parity errors (max over the comparisons of each test)")
    for test, e in sorted(worst.items()):
        terminalreporter.write_line("%.3e  %s" % (e, test))
    path = os.environ.get("GDN_PARITY_LOG")
    if path:
        import json
        with open(path, "a") as f:
            for test, e in sorted(worst.items()):
                f.write(json.dumps({"test": test, "max_rel_err": e}) + "\n")
