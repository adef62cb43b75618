"""Shared pytest set-up: the ``gpu`` marker and the repository root on sys.path."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")


import pytest  # noqa: E402


@pytest.fixture(params=["streaming", "registers"])
def family(request):
    """Runs a test once with the shared-memory streaming kernels and once with
    the register kernels (the library's two kernel families)."""
    import swiglu_ar_tts_b200 as ops

    old = ops.set_streaming(request.param == "streaming")
    yield request.param
    ops.set_streaming(old)


@pytest.fixture(autouse=True)
def _no_device_errors(request):
    """Every GPU test must leave the library's device error word at 0 (no
    bounded wait in any kernel ran out)."""
    yield
    if request.node.get_closest_marker("gpu") is None:
        return
    import torch

    import swiglu_ar_tts_b200 as ops

    if torch.cuda.is_available():
        torch.cuda.synchronize()
        assert ops.device_errors(clear=True) == 0


@pytest.fixture(scope="session", autouse=True)
def _built_libraries():
    """Compile libarops.so (nvcc, sm_100a) and the C oracle if they are missing
    or older than their sources, so every test runs against the current code."""
    from swiglu_ar_tts_b200 import build

    import oracle

    build.build()
    oracle.build()
    oracle.build(omp=True)
