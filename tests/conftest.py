import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")
    # the package loads libmsa.so on import: (re)build it first when it is missing or older than its
    # sources (nvcc cross-compiles for sm_100a without a GPU); the builder is loaded by path so that
    # no stale library gets imported on the way
    import importlib.util

    spec = importlib.util.spec_from_file_location("msa_build", os.path.join(ROOT, "routed_long_context_b200",
                                                                            "build.py"))
    builder = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(builder)
    builder.build()
