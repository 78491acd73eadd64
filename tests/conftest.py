import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_terminal_summary(terminalreporter):
    """The parity margins recorded by tests.helpers.margin: for each check,
    the largest max |gpu - oracle| seen and its share of the tolerance."""
    helpers = sys.modules.get("tests.helpers")
    rows = getattr(helpers, "MARGINS", None)
    if not rows:
        return
    worst = {}
    for what, qty, err, tol in rows:
        key = (what, qty)
        if key not in worst or err / tol > worst[key][0] / worst[key][1]:
            worst[key] = (err, tol)
    tr = terminalreporter
    ranked = sorted(worst.items(), key=lambda kv: -kv[1][0] / kv[1][1])
    shown = ranked[:30]
    tr.write_sep("-", f"parity margins: max |gpu - reference| / tolerance, the {len(shown)} tightest of "
                      f"{len(worst)} checks")
    for (what, qty), (err, tol) in shown:
        tr.write_line(f"{err / tol:7.1%}  {qty:<4} {err:.2e} <= {tol:.1e}  {what}")
    if len(ranked) > len(shown):
        tr.write_line(f"the other {len(ranked) - len(shown)} checks use at most "
                      f"{ranked[len(shown)][1][0] / ranked[len(shown)][1][1]:.1%} of their tolerance")
