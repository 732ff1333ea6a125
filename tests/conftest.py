import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def _build_libraries():
    """Build the CUDA library and the generator library in-tree if missing or
    stale (nvcc cross-compiles for sm_100a without a GPU)."""
    import gen.build
    import oracle.build
    import sparse_moe_layer_renormalised_b200.build as b

    b.build()
    oracle.build.build()
    if not os.path.exists(os.path.join(ROOT, "gen", "libmoegen.so")):
        gen.build.build()


def pytest_configure(config):
    _build_libraries()
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (sm_100a); run with -m gpu")
    config.addinivalue_line("markers", "slow: long-running check at the full K3 sizes")


def pytest_collection_modifyitems(config, items):
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


def read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            rows.append(line.split())
    return rows
