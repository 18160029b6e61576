"""Worst parity errors per test, printed at the end of a pytest run (conftest.py).

Each record is (test id, what, out max-abs, out mean-abs, lse max-abs); the
summary shows how close each test came to its tolerance, so drift toward a limit
is visible before a test fails.
"""
import os

RECORDS = []


def record(what, out_max, out_mean, lse_max):
    test = os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0]
    RECORDS.append((test, what, float(out_max), float(out_mean), float(lse_max)))


def summary_lines(out_max_tol, out_mean_tol, lse_tol, top=12):
    """One line per test: its worst case as a fraction of each tolerance, worst tests first."""
    worst = {}
    for test, what, a, b, c in RECORDS:
        frac = max(a / out_max_tol, b / out_mean_tol, c / lse_tol)
        if test not in worst or frac > worst[test][0]:
            worst[test] = (frac, what, a, b, c)
    rows = sorted(worst.items(), key=lambda kv: -kv[1][0])
    lines = [f"parity headroom: {len(RECORDS)} comparisons in {len(worst)} tests; worst fraction of a tolerance "
             f"(out max {out_max_tol:g}, out mean {out_mean_tol:g}, lse {lse_tol:g}):"]
    for test, (frac, what, a, b, c) in rows[:top]:
        lines.append(f"  {frac:5.2f}  max {a:.2e} mean {b:.2e} lse {c:.2e}  {test.split('::')[-1]} [{what}]")
    return lines
