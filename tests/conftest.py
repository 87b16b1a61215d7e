import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: long CPU test")


def pytest_collection_modifyitems(config, items):
    """GPU tests are skipped (not failed) when no CUDA device is present and
    they were not explicitly requested with -m gpu."""
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    markexpr = config.getoption("-m") or ""
    if has_gpu or "gpu" in markexpr and "not gpu" not in markexpr:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)


def pytest_terminal_summary(terminalreporter):
    """Accuracy of the INT4 path on the GPU parity cases: max-abs error against
    the oracle, error relative to the row norm, cosine against unquantised
    attention."""
    try:
        import gpu_util
    except Exception:
        return
    if not gpu_util.ACCURACY:
        return
    terminalreporter.write_sep("-", "INT4 accuracy (vs oracle; cosine vs unquantised attention)")
    for name, r in gpu_util.ACCURACY:
        terminalreporter.write_line(
            f"{name:40s} max_abs {r['max_abs_vs_oracle']:.3e}  rel_row_norm {r['max_rel_row_norm']:.3e}  "
            f"cos_unq mean {r['cos_vs_unquantised_mean']:.4f} min {r['cos_vs_unquantised_min']:.4f}  "
            f"rows {r['rows']}")
