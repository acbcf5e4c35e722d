import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")


def pytest_collection_modifyitems(config, items):
    # A GPU test run on a machine without a GPU is a setup error, not a skip:
    # the product path has no CPU fallback.  Tests select with -m gpu / -m "not gpu".
    pass


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Largest error of each output kind per workload, against the oracle, with the share of
    the bound it used (bf16: O within 2e-2; gradients within 2e-2 beyond their own bf16
    rounding; float32: relative to the tensor's largest entry, within 1e-4)."""
    try:
        from tests.harness import RECORDS
    except Exception:
        return
    if not RECORDS:
        return
    worst = {}
    for test, wl, name, err, used in RECORDS:
        kind = name.split("[")[0].split(" ")[0]
        key = (wl, kind)
        if key not in worst or used > worst[key][1]:
            worst[key] = (err, used, test)
    tr = terminalreporter
    tr.write_sep("-", "largest error against the float64 oracle, per workload and output")
    for (wl, kind), (err, used, test) in sorted(worst.items()):
        tr.write_line(f"{wl:58s} {kind:8s} max err {err:.3e}  bound used {100 * used:5.1f}%  ({test})")
