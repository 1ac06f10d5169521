"""pytest configuration: the ``gpu`` marker and shared helpers.

``-m "not gpu"`` runs everywhere (oracle pins, host logic, symbol exports);
``-m gpu`` needs a B200 and the built CUDA library.
"""

import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (sm_100a) and the built library")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA GPU in this environment")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


@pytest.fixture(params=["tile_per_cta", "persistent"])
def tiled_path(request):
    """Run the transposed / dual quantize on each of its two kernels: one tile per CTA, or
    the persistent TMA-fed kernel (forced by a zero tile threshold)."""
    import fp8_delayed_scaling_amax_b200 as F
    F.fp8_set_tiled_persist_threshold(0 if request.param == "persistent" else 1 << 40)
    yield request.param
    F.fp8_set_tiled_persist_threshold(1024)
