import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_addoption(parser):
    parser.addoption("--full-oracle", action="store_true", default=False,
                     help="run the full_oracle tests: every row of the largest packs against "
                          "the fp64 oracle (about 15 min of host CPU per pack)")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU")
    config.addinivalue_line("markers", "slow: longer CPU test")
    config.addinivalue_line("markers", "full_oracle: needs a B200 and --full-oracle (long oracle run)")


def pytest_collection_modifyitems(config, items):
    # GPU tests are skipped (not failed) when no GPU is visible, so that
    # `-m "not gpu"` and plain runs work on CPU-only machines.
    # full_oracle tests are not marked gpu (so `-m gpu` leaves them out) and
    # run only when asked for with --full-oracle, on a GPU.
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    full = config.getoption("--full-oracle")
    skip_full = pytest.mark.skip(reason="needs --full-oracle and a CUDA device")
    for item in items:
        if "full_oracle" in item.keywords and not (full and has_gpu):
            item.add_marker(skip_full)
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device visible")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)
