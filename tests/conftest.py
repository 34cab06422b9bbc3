import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workloads")


def _ensure_built():
    """Build librtp.so (nvcc), the oracle and the generator if missing or stale."""
    import importlib.util

    spec = importlib.util.spec_from_file_location(
        "_rtp_build", os.path.join(ROOT, "sparse_attention_decode_rtpurbo_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()


_ensure_built()
