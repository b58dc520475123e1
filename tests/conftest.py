import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200) and the built liblh.so")
    config.addinivalue_line("markers", "slow: full-size workload, minutes of CPU time for the oracle")


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Print the achieved parity errors of every float comparison the run made
    (max-abs, mean-abs, and each as a fraction of its bound), and write them as
    JSON lines to $LH_PARITY_LOG when that is set."""
    mod = sys.modules.get("tests.parity_util")
    rows = getattr(mod, "RESULTS", None) if mod else None
    if not rows:
        return
    tr = terminalreporter
    tr.section("parity errors (bound: |err| <= 2e-2 + half an ulp of the stored dtype; mean <= 2e-3 + mean half ulp)")
    tr.write_line(f"{'check':70s} {'dtype':5s} {'max-abs':>10s} {'of bound':>8s} {'mean-abs':>10s} {'of bound':>8s} "
                  f"{'max-abs |x|<=1':>14s}")
    for r in rows:
        tag = "" if r["kind"] == "check" else "  (info)"
        tr.write_line(f"{r['name'][:70]:70s} {r['dtype']:5s} {r['max_abs']:10.3e} {r['max_ratio']:8.3f} "
                      f"{r['mean_abs']:10.3e} {r['mean_ratio']:8.3f} {r.get('max_abs_unit', 0.0):14.3e}{tag}")
    path = os.environ.get("LH_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            for r in rows:
                f.write(json.dumps(r) + "\n")
