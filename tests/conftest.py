import os
import shutil
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    # Build the oracle (gcc) and the CUDA library (nvcc cross-compiles without a
    # GPU); both builds are skipped when the shared objects are up to date.
    import oracle
    oracle.build()
    if shutil.which(os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")) or \
            os.path.exists("/usr/local/cuda/bin/nvcc"):
        from speculative_decoding_rl_b200 import build
        build.build()


def cuda_available() -> bool:
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


def pytest_collection_modifyitems(config, items):
    if cuda_available():
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)
