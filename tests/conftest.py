"""Shared pytest configuration.

Marker ``gpu``: the test needs a B200 (sm_100a) and the built CUDA library.
``python -m pytest -m "not gpu"`` runs the CPU suite (oracle pins, host
logic, library load / symbol checks); ``-m gpu`` runs the parity tests.
"""

import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def pytest_collection_modifyitems(config, items):
    # A GPU test on a machine without a GPU is an error in the caller's
    # selection, not something to skip silently: fail loudly.
    pass


def _ensure_library_built():
    """Build libmxq.so in-tree when it is missing or older than its sources
    (loads the build script by path: importing the package needs the library)."""
    import importlib.util
    path = os.path.join(ROOT, "fp8_gemm_diffusion_b200", "build.py")
    spec = importlib.util.spec_from_file_location("_mxq_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()


_ensure_library_built()
