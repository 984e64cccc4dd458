import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(ROOT, "tests", "golden")


def pytest_terminal_summary(terminalreporter):
    """Parity records of the tests that compared the device with the oracle: units,
    steps, compressions, near-tie units and the largest errors of the units compared
    in full (relative Frobenius)."""
    mod = sys.modules.get("parity_util")
    rows = getattr(mod, "SUMMARY", None) if mod is not None else None
    if not rows:
        return
    tr = terminalreporter
    tr.section("parity against the fp64 oracle")
    tot_units = sum(r["units"] for r in rows)
    tot_ties = sum(r["near_ties"] for r in rows)
    fmt = lambda x: "-" if x is None else f"{x:.1e}"  # noqa: E731
    for r in rows:
        tr.write_line(f"{r['label']}: {r['units']} units x {r['steps']} steps, {r['compressions']} "
                      f"compressions, near-ties {r['near_ties']}, max err o {fmt(r['max_err_o'])} "
                      f"S {fmt(r['max_err_S'])} sigma {fmt(r['max_err_sigma'])}, compressions checked "
                      f"optimal {r['compressions_checked']}")
    tr.write_line(f"total: {tot_units} units compared, {tot_ties} near-ties "
                  f"({100.0 * tot_ties / max(tot_units, 1):.2f} %)")
