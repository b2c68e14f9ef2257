import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (sm_100a) and the built CUDA library")


def pytest_collection_modifyitems(config, items):
    # GPU tests fail loudly (not skip) when the device is missing but a GPU run was asked for;
    # in a CPU-only run they are deselected with -m "not gpu".
    pass


def pytest_terminal_summary(terminalreporter):
    # achieved errors of every parity comparison that ran (see tests/_parity.py)
    try:
        import _parity
    except ImportError:
        return
    recs = _parity.RECORDS
    if not recs:
        return
    tr = terminalreporter
    tr.write_sep("-", f"parity: achieved errors ({len(recs)} comparisons)")
    worst = max((r for r in recs if r["kind"] != "exact"), key=lambda r: r["rel_err"] / r["tol"], default=None)
    n_exact = sum(r["kind"] == "exact" for r in recs)
    for r in recs:
        if r["kind"] == "exact":
            tr.write_line(f"  exact  {r['case']}: {r['mismatches']} of {r['elements']} elements differ")
        else:
            tr.write_line(f"  {r['rel_err']:.2e} (tol {r['tol']:.0e}, max/rms {r['max_over_rms']:.2e})  {r['case']}")
    if worst:
        tr.write_line(f"  worst rel_err/tol: {worst['rel_err'] / worst['tol']:.3f} ({worst['case']}); "
                      f"{n_exact} bit-exact comparisons")
    path = os.environ.get("EQLIN_PARITY_LOG")
    if path:
        import json
        with open(path, "w") as f:
            json.dump(recs, f, indent=1)


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.build()
    return oracle
