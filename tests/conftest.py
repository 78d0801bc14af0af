import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the CUDA library")


def pytest_collection_modifyitems(config, items):
    # GPU tests fail loudly when the device is missing; they never fall back.
    pass


@pytest.fixture(autouse=True)
def _no_index_out_of_bounds():
    """Under the bounds-checking build (NVFP4_LIBRARY=debug), fail a test
    after which the device status word reads NVFP4_ERR_BOUNDS (8)."""
    yield
    if os.environ.get("NVFP4_LIBRARY") != "debug":
        return
    import torch
    if not torch.cuda.is_available():
        return
    import qad_nvfp4_quantize_b200 as nv
    st = nv.device_status(clear=True)
    assert st != 8, "the bounds-checking build flagged an index outside its buffer"


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(ROOT, "tests", "golden")
