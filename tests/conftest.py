import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_terminal_summary(terminalreporter):
    """Kept-set agreement of every GPU parity check of the run (lane-levels compared, exact,
    logged mass / score near-ties) and the output errors, one line each."""
    tl = sys.modules.get("zha_testlib")
    log = getattr(tl, "TIE_LOG", None) if tl else None
    notes = getattr(tl, "NOTES", None) if tl else None
    if notes:
        terminalreporter.section("measured rates")
        for line in notes:
            terminalreporter.write_line(line)
    if not log:
        return
    tr = terminalreporter
    tr.section("kept-set parity: lane-levels, exact, logged near-ties, output errors")
    tot = [0, 0, 0, 0]
    for name, lv, ex, mt, st, e1, e2 in log:
        tr.write_line("%-40s levels=%6d exact=%6d mass_ties=%3d score_ties=%3d  err/own=%.2e err/e2e=%.2e"
                      % (name[:40], lv, ex, mt, st, e1, e2))
        tot = [tot[0] + lv, tot[1] + ex, tot[2] + mt, tot[3] + st]
    tr.write_line("total: %d lane-levels, %d exact, %d mass ties, %d score ties (tie rate %.3f%%)"
                  % (tot[0], tot[1], tot[2], tot[3], 100.0 * (tot[2] + tot[3]) / max(1, tot[0])))
