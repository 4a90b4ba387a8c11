"""Shared pytest configuration.

Markers:
  gpu -- needs a CUDA device (B200, sm_100a); everything else runs on CPU.
"""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: test needs a CUDA GPU (sm_100a)")


@pytest.fixture(scope="session")
def orc():
    alt = os.environ.get("FP8Q_ORACLE_DIR")
    if alt:
        # a copy of the oracle with one planted mistake (tests/test_oracle_mutations.py)
        import importlib.util
        spec = importlib.util.spec_from_file_location("oracle_under_test", os.path.join(alt, "__init__.py"),
                                                      submodule_search_locations=[alt])
        oracle = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(oracle)
    else:
        import oracle
    oracle.build()
    oracle.lib()
    return oracle


@pytest.fixture(scope="session")
def fp8q():
    """The CUDA library's Python binding, built for sm_100a (rebuilt if stale)."""
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from dequantisation_fp8q_token_b200 import build as _build
    _build.build()
    import dequantisation_fp8q_token_b200 as m
    m.lib()
    return m
