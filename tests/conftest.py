import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built libmetis")
    config.addinivalue_line("markers", "slow: long CPU test (full-size oracle work)")


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(ROOT, "tests", "golden")


@pytest.fixture(scope="session")
def metis_lib():
    """The libmetis binding, building the library first if it is missing or stale."""
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_metis_build", os.path.join(ROOT, "spectral_quantized_gemm_b200", "build.py"))
    builder = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(builder)
    builder.build()
    import spectral_quantized_gemm_b200 as lib
    return lib


@pytest.fixture(scope="session")
def ctx(metis_lib):
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    c = metis_lib.Context()
    yield c
    c.close()
