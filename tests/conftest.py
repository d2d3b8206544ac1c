import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
# The oracle's planted-mistake tests run the pins in a subprocess against a modified copy of
# the oracle package placed in this directory; it is registered as `oracle` before any test
# module imports that name.
if os.environ.get("NQ_ORACLE_PKG_DIR"):
    import importlib.util

    _pkg = os.path.join(os.environ["NQ_ORACLE_PKG_DIR"], "oracle")
    _spec = importlib.util.spec_from_file_location("oracle", os.path.join(_pkg, "__init__.py"),
                                                   submodule_search_locations=[_pkg])
    _mod = importlib.util.module_from_spec(_spec)
    sys.modules["oracle"] = _mod
    _spec.loader.exec_module(_mod)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100) GPU and the CUDA library")


def load_golden(name):
    """Parses a tests/golden text fixture: 'key: values' lines, rows split by ';'."""
    out = {}
    with open(os.path.join(ROOT, "tests", "golden", name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, _, val = line.partition(":")
            rows = [r.split() for r in val.split(";")]
            out[key.strip()] = rows if len(rows) > 1 else rows[0]
    return out


def pytest_terminal_summary(terminalreporter):
    """Numerical headroom of the parity checks that ran (GPU runs only)."""
    mod = sys.modules.get("tests.gpu_util")
    rows = getattr(mod, "MARGINS", None) if mod else None
    if not rows:
        return
    tr = terminalreporter
    tr.section("parity headroom: max |err|/tol (tol with half a bf16 ulp) and max |err|/(2e-3 S + 1e-5)")
    for what, ratio, strict in rows:
        tr.write_line("%-60s %8.4f %8.4f" % (what[:60], ratio, strict))
    out = os.environ.get("NQ_MARGINS_JSON")
    if out:
        import json
        with open(out, "w") as f:
            json.dump([{"check": w, "err_over_tol": r, "err_over_strict_bound": s} for w, r, s in rows], f, indent=1)
