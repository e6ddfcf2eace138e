import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU")
    # The CUDA library is not kept in git; build it (incrementally) before any
    # test imports the binding.  nvcc cross-compiles without a GPU.
    from flash_attention_tiled_b200 import build
    build.build()
