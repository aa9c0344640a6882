import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the CUDA library")


def pytest_collection_modifyitems(config, items):
    # GPU tests are skipped cleanly when no GPU is visible (the CPU suite is run
    # with -m "not gpu"; this guard only matters for an unfiltered run here).
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device visible")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """The achieved parity errors of the GPU tests (worst per test), beside the tolerances
    they are held to: max-rel of o <= 1e-4 (fp32 mode) / 2e-2 (bf16), rel-L2 of S_T <= 1e-2."""
    try:
        import parity_util as U
    except Exception:
        return
    if not U.MARGINS:
        return
    tr = terminalreporter
    tr.write_sep("-", "achieved parity errors (worst per test)")
    for test in sorted(U.MARGINS):
        ent = U.MARGINS[test]
        cols = "  ".join(f"{k}={v:.3e}" for k, v in sorted(ent.items()))
        tr.write_line(f"{cols}  {test}")
    path = os.environ.get("GDR_PARITY_LOG")
    if path:
        U.write_margins(path)
