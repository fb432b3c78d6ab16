import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a) and the built libkin.so")


def pytest_collection_modifyitems(config, items):
    # GPU tests cannot run without a device; skip them cleanly on CPU hosts.
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """How often a GPU top-k set differed from the oracle's and was accepted
    as a near tie (kin_tiecheck), per test that compared selections."""
    mod = sys.modules.get("kin_tiecheck")
    if mod is None or not mod.TALLY:
        return
    tally = {k: v for k, v in mod.TALLY.items() if "test_tiecheck" not in k}
    if not tally:
        return
    tr = terminalreporter
    tr.write_sep("-", "top-k sets compared with the oracle / accepted near ties")
    total = [0, 0]
    for name, (n, d) in sorted(tally.items()):
        tr.write_line(f"{name}: {n} compared, {d} near-tie")
        total[0] += n
        total[1] += d
    tr.write_line(f"all: {total[0]} compared, {total[1]} near-tie")
