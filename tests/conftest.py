import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running case")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA GPU in this environment")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)


def pytest_terminal_summary(terminalreporter):
    """Prints every recorded parity error (achieved rel-L2 next to its
    tolerance); with KDA_MARGINS_FILE set, also writes them there as TSV."""
    mod = sys.modules.get("kda_testutil")
    rows = getattr(mod, "MARGINS", []) if mod is not None else []
    if not rows:
        return
    tr = terminalreporter
    tr.section("parity margins (achieved rel-L2 / tolerance)")
    worst = max(rows, key=lambda r: r[2] / r[3])
    for test, what, e, tol in rows:
        tr.write_line(f"{e:10.3e} / {tol:g}  {test}  {what}")
    tr.write_line(f"{len(rows)} comparisons; largest fraction of the tolerance: {worst[2] / worst[3]:.3f} "
                  f"({worst[0]} {worst[1]})")
    path = os.environ.get("KDA_MARGINS_FILE")
    if path:
        with open(path, "w") as f:
            f.write("test\tquantity\trel_l2\ttolerance\n")
            for test, what, e, tol in rows:
                f.write(f"{test}\t{what}\t{e:.6e}\t{tol:g}\n")
