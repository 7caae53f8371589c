import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: long-running CPU check")


# The forward's acceptance checks run before the paths built on top of it, so
# that a failure in an extension (under -x) cannot hide them; the static-
# workspace file stays last, as its name intends.  The sort is stable.
_GPU_ORDER = ["test_gpu_parity", "test_gpu_prepare", "test_gpu_segmented", "test_gpu_epilogue",
              "test_gpu_momentum", "test_gpu_two_pass_simt", "test_gpu_vjp", "test_gpu_timeout"]


def pytest_collection_modifyitems(session, config, items):
    def rank(item):
        name = os.path.splitext(os.path.basename(str(item.fspath)))[0]
        if name in _GPU_ORDER:
            return (1, _GPU_ORDER.index(name))
        return (2, 0) if name.startswith("test_zz") else (0, 0)

    items.sort(key=rank)
