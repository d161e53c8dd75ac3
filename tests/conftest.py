import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a) and the built library")
    config.addinivalue_line("markers", "slow: full-size workload test")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Prints the error figures of every GPU comparison of the run (tests/_gpu.py REPORT)."""
    mod = sys.modules.get("_gpu")
    rows = getattr(mod, "REPORT", None) if mod else None
    if not rows:
        return
    tr = terminalreporter
    tr.write_sep("-", "GPU parity figures (normwise rel, MAE, MAE/mean|o|, element-wise max and p99 where |o| > 0.1 rms)")
    for what, dtype, f in rows:
        tr.write_line(f"{what[:58]:58s} {dtype:4s} rel {f['rel']:.2e}  mae {f['mae']:.2e}  mae_rel {f['mae_rel']:.2e}"
                      f"  elem_max {f['elem_max']:.2e}  elem_p99 {f['elem_p99']:.2e}  n={f['n']}")
