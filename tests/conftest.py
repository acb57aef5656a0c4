import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _ensure_library_built():
    """Compile libpace.so in-tree if it is missing or older than its sources
    (the build script runs without importing the package)."""
    import subprocess
    script = os.path.join(ROOT, "bit_recurrent_state_pace_b200", "build.py")
    subprocess.run([sys.executable, script], check=True, stdout=subprocess.DEVNULL)


def pytest_configure(config):
    _ensure_library_built()
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: longer CPU test")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA GPU in this environment")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)
