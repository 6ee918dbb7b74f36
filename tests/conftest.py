import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def gpu_available():
    try:
        import torch

        return torch.cuda.is_available()
    except Exception:
        return False


def pytest_collection_modifyitems(config, items):
    if gpu_available():
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    # parity margins recorded by the GPU tests (tests/_helpers.record_parity), printed so that
    # every run's log shows how much of each tolerance was used
    from tests._helpers import PARITY_RECORDS

    if not PARITY_RECORDS:
        return
    tr = terminalreporter
    tr.section("parity margins (GPU vs fp64 oracle)")
    tr.write_line(f"{'case':<58} {'max_rel_err':>11} {'of 2e-3':>7} {'excluded':>9} {'codes':>10} "
                  f"{'norm_ulp':>8}")
    for r in PARITY_RECORDS:
        err = r.get("max_rel_err")
        tr.write_line(
            f"{r['case'][:58]:<58} {('%.3e' % err) if err is not None else '-':>11} "
            f"{('%.0f%%' % (100 * err / 2e-3)) if err is not None else '-':>7} "
            f"{r.get('excluded', '-')!s:>9} {r.get('codes', '-')!s:>10} {r.get('norm_ulp', '-')!s:>8}")
