import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_terminal_summary(terminalreporter):
    """Prints the achieved maximum errors of every parity check that ran."""
    from tests import parity
    if not parity.RECORD:
        return
    tr = terminalreporter
    tr.section("parity: achieved max errors (O max-abs, worst error / bound, LSE max-abs)")
    worst = max(r[2] for r in parity.RECORD)
    for what, o_err, ratio, l_err in parity.RECORD:
        tr.write_line("%-90.90s  O %.3e  %.3f  LSE %.3e" % (what, o_err, ratio, l_err))
    tr.write_line("%d checks; largest O error / bound %.3f; largest LSE error %.3e" % (
        len(parity.RECORD), worst, max(r[3] for r in parity.RECORD)))
